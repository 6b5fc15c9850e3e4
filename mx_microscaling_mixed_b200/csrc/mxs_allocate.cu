// mxs_allocate.cu -- 4/6/8-bit allocation and column permutation.
//
// MXSens (arXiv 2607.17733), technical summary §2.3 (sensitivity-guided
// allocation): per linear layer the columns are sorted by sensitivity; the 32
// most sensitive always get 8-bit mantissas (one MXINT block, §2.2); a
// sensitivity-driven number of columns get 6 bits so that a global average
// budget B is met; the rest get 4 bits.  §4: at ~4.03 bits about 1% of the
// work is at higher precision (4 + 4*32/4096 = 4.03125 for K = 4096).
//
// Fixed readings: ranking by s descending with ties to the lower column;
// budget = average mantissa bits over all weight elements (scales excluded);
// the 6-bit count comes from a greedy over 32-column groups ordered by
// gain/cost across layers (gain = layer weight x summed s, cost = 2 N count
// bits), stopping at the first group that does not fit.
//
// Device work: an all-pairs rank count (each CTA ranks 32 columns against
// every candidate, 32 threads per column each taking a slice of every
// candidate tile staged in shared memory, partial counts added in shared
// memory -- exact and order-free, no atomics), the group gains (one thread
// sums one group in rank order), and a stable compaction that writes the
// permutation segment by segment in ascending column order (each CTA counts
// the segments of all columns before its range, then scans its own).  The integer budget
// arithmetic and the cross-layer greedy are a few hundred scalar steps and
// run on the host side of the call; only the multi-layer greedy needs device
// data (the group gains) and so a stream synchronisation.
#include <algorithm>
#include <cmath>
#include <vector>

#include "mxs_internal.cuh"

namespace mxs {

constexpr int kRankCols = 32;                     // columns ranked per CTA
constexpr int kRankParts = 32;                    // candidate slices per column
constexpr int kRankThreads = kRankCols * kRankParts;
constexpr int kRankTile = 4096;                   // candidates staged per pass (32 KB)
constexpr int kRankSlice = kRankTile / kRankParts;

// rank[j] = #{i : s_i > s_j, or s_i == s_j and i < j}.  Thread (part, c)
// counts candidate slice `part` of every tile for column j = 32 blockIdx.x + c.
// Slices wholly before j count ties, slices wholly after j do not; only the
// slice holding j compares indices.
__global__ void __launch_bounds__(kRankThreads) rank_kernel(const double *s, int64_t K, int32_t *rank) {
  pdl_wait();
  pdl_trigger();
  __shared__ double tile[kRankTile];
  __shared__ int part_cnt[kRankParts][kRankCols];
  const int c = threadIdx.x % kRankCols, part = threadIdx.x / kRankCols;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * kRankCols + c;
  const double sj = j < K ? s[j] : 0.0;
  int r = 0;
  for (int64_t base = 0; base < K; base += kRankTile) {
    const int n = static_cast<int>(min(static_cast<int64_t>(kRankTile), K - base));
    __syncthreads();
    {
      // every thread's loads in flight together, then the stores
      constexpr int kPer = kRankTile / kRankThreads;
      double v[kPer];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int i = threadIdx.x + u * kRankThreads;
        v[u] = i < n ? s[base + i] : 0.0;
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int i = threadIdx.x + u * kRankThreads;
        if (i < n) tile[i] = v[u];
      }
    }
    __syncthreads();
    const int i0 = part * kRankSlice, i1 = min(i0 + kRankSlice, n);
    if (base + i1 <= j) {
#pragma unroll 8
      for (int i = i0; i < i1; ++i) r += tile[i] >= sj;
    } else if (base + i0 > j) {
#pragma unroll 8
      for (int i = i0; i < i1; ++i) r += tile[i] > sj;
    } else {
      for (int i = i0; i < i1; ++i) {
        const double si = tile[i];
        r += (si > sj) | ((si == sj) & (base + i < j));
      }
    }
  }
  part_cnt[part][c] = r;
  __syncthreads();
  if (threadIdx.x < kRankCols && j < K) {
    int tot = 0;
#pragma unroll
    for (int q = 0; q < kRankParts; ++q) tot += part_cnt[q][threadIdx.x];
    rank[j] = tot;
  }
}

__global__ void order_kernel(const int32_t *rank, int64_t K, int32_t *order) {
  pdl_wait();
  pdl_trigger();
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j < K) order[rank[j]] = static_cast<int32_t>(j);
}

// gains[g] = sum of s over ranks [n8 + 32 g, min(n8 + 32 g + 32, K)), in rank order.
__global__ void group_gain_kernel(const double *s, const int32_t *order, int64_t K, int64_t n8,
                                  int64_t ngroups, double *gains) {
  pdl_wait();
  pdl_trigger();
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= ngroups) return;
  const int64_t r0 = n8 + 32 * g, r1 = min(r0 + 32, K);
  double sum = 0.0;
  for (int64_t r = r0; r < r1; ++r) sum = __dadd_rn(sum, s[order[r]]);
  gains[g] = sum;
}

// The permutation: a stable compaction by segment.  CTA c places columns
// [256 c, 256 c + 256).  Its threads first count, over all columns before
// the CTA's range, how many fall in segments 0 and 1 (two 32-bit fields of
// a 64-bit word, loads batched 8 per thread, a block reduction); a block
// scan over its own columns then gives each one its slot.  The permutation keeps
// ascending column order inside each segment.
constexpr int kPlaceCols = 256;

__device__ __forceinline__ unsigned long long seg_word(int64_t r, int64_t n8, int64_t n6) {
  return r < n8 ? 1ull : (r < n8 + n6 ? (1ull << 32) : 0ull);
}

__global__ void __launch_bounds__(kPlaceCols) perm_place_kernel(const int32_t *rank, int64_t K, int64_t n8,
                                                               int64_t n6, int32_t *perm) {
  pdl_wait();
  pdl_trigger();
  __shared__ unsigned long long warp_tot[kPlaceCols / 32];
  __shared__ unsigned long long before_cta;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kPlaceCols;
  // segment counts over columns [0, c0)
  unsigned long long cnt = 0;
  for (int64_t j0 = threadIdx.x; j0 < c0; j0 += 8 * kPlaceCols) {
    int32_t r[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t j = j0 + static_cast<int64_t>(u) * kPlaceCols;
      r[u] = j < c0 ? rank[j] : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (r[u] >= 0) cnt += seg_word(r[u], n8, n6);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) warp_tot[warp] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long t = 0;
    for (int w = 0; w < kPlaceCols / 32; ++w) t += warp_tot[w];
    before_cta = t;
  }
  __syncthreads();
  // this CTA's columns: an exclusive block scan of their segment words
  const int64_t j = c0 + threadIdx.x;
  const int64_t rj = j < K ? rank[j] : -1;
  const unsigned long long mine = rj >= 0 ? seg_word(rj, n8, n6) : 0ull;
  unsigned long long inc = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  unsigned long long wbefore = 0;
  for (int w = 0; w < warp; ++w) wbefore += warp_tot[w];
  if (rj < 0) return;
  const unsigned long long before = before_cta + wbefore + inc - mine;
  const int64_t b0 = static_cast<int64_t>(before & 0xFFFFFFFFull), b1 = static_cast<int64_t>(before >> 32);
  int64_t slot;
  if (rj < n8) slot = b0;
  else if (rj < n8 + n6) slot = n8 + b1;
  else slot = n8 + n6 + (j - b0 - b1);
  perm[slot] = static_cast<int32_t>(j);
}

struct LayerWs {
  int32_t *rank;
  int32_t *order;
  double *gains;
};

static size_t layer_ws_bytes(int64_t K) {
  const int64_t ng = K / 32 + 2;
  return static_cast<size_t>(round_up(K * 4, 256) * 2 + round_up(ng * 8, 256));
}

static int64_t round_half_up_frac(int64_t num, int64_t den, int64_t K) {
  return (2 * num * K + den) / (2 * den);
}

}  // namespace mxs

using namespace mxs;

extern "C" mxs_status mxs_allocate_workspace_bytes(int32_t n_layers, const int64_t *K, size_t *bytes) {
  if (n_layers < 1 || !K || !bytes) return MXS_ERR_ARG;
  size_t b = 0;
  for (int l = 0; l < n_layers; ++l) {
    if (K[l] < 1) return MXS_ERR_ARG;
    b += layer_ws_bytes(K[l]);
  }
  *bytes = b;
  return MXS_OK;
}

// Budget mode: the bit budget (num/den bits per weight over all layers)
// times den, and what the 4-bit columns plus the fixed 8-bit block already
// use of it.  Infeasible when used > cap.
static void budget_base(int32_t n_layers, const int64_t *K, const int64_t *N, const mxs_budget &B, __int128 &cap,
                        __int128 &used) {
  cap = 0;
  used = 0;
  for (int l = 0; l < n_layers; ++l) {
    const int64_t n8 = std::min<int64_t>(B.fixed8, K[l]);
    cap += static_cast<__int128>(B.num) * N[l] * K[l];
    used += static_cast<__int128>(B.den) * N[l] * (4 * K[l] + 4 * n8);
  }
}

// The layer-score rule: layer l with score w_l > 0 reaches its k-th
// 32-column 6-bit group at R = 32 k / w_l.  Steps are ordered by that R,
// compared exactly (k_a w_b against k_b w_a, each product as the pair of its
// rounded value and its fma rounding error, compared lexicographically), and
// taken in increasing R, all steps of one R value together, while they fit.
struct RStep {
  int32_t layer;
  int64_t k, cols;
};

static int rstep_cmp(const RStep &a, const RStep &b, const double *w) {
  const double ka = static_cast<double>(a.k), kb = static_cast<double>(b.k);
  const double p1 = ka * w[b.layer], e1 = std::fma(ka, w[b.layer], -p1);
  const double p2 = kb * w[a.layer], e2 = std::fma(kb, w[a.layer], -p2);
  if (p1 != p2) return p1 < p2 ? -1 : 1;
  if (e1 != e2) return e1 < e2 ? -1 : 1;
  return 0;
}

static void layer_rule(int32_t n_layers, const int64_t *K, const int64_t *N, const double *w, const mxs_budget &B,
                       const std::vector<int64_t> &n8, __int128 cap, __int128 used, std::vector<int64_t> &n6) {
  std::vector<RStep> st;
  for (int l = 0; l < n_layers; ++l) {
    if (!(w[l] > 0.0)) continue;
    const int64_t avail = K[l] - n8[l];
    for (int64_t k = 1; 32 * (k - 1) < avail; ++k) st.push_back(RStep{l, k, std::min<int64_t>(32, avail - 32 * (k - 1))});
  }
  std::sort(st.begin(), st.end(), [w](const RStep &a, const RStep &b) { return rstep_cmp(a, b, w) < 0; });
  for (size_t a = 0; a < st.size();) {
    size_t b = a + 1;
    while (b < st.size() && rstep_cmp(st[a], st[b], w) == 0) ++b;
    __int128 add = 0;
    for (size_t j = a; j < b; ++j) add += static_cast<__int128>(B.den) * 2 * N[st[j].layer] * st[j].cols;
    if (used + add > cap) break;                     // R stays below this step value
    used += add;
    for (size_t j = a; j < b; ++j) n6[st[j].layer] += st[j].cols;
    a = b;
  }
}

extern "C" mxs_status mxs_allocate(int32_t n_layers, const int64_t *K, const int64_t *N,
                                   const double *const *s, const double *layer_w,
                                   const mxs_budget *budget, int32_t *const *perm,
                                   int64_t *counts, void *ws, size_t ws_bytes, void *stream) {
  if (n_layers < 1 || !K || !N || !s || !budget || !perm || !counts) return MXS_ERR_ARG;
  for (int l = 0; l < n_layers; ++l) {
    if (K[l] < 1 || N[l] < 1 || !s[l] || !perm[l]) return MXS_ERR_ARG;
    if (K[l] > INT32_MAX) return MXS_ERR_SHAPE;
  }
  const mxs_budget &B = *budget;
  if (B.mode == MXS_ALLOC_FRACTIONS) {
    if (B.p8_den <= 0 || B.p6_den <= 0 || B.p8_num < 0 || B.p6_num < 0) return MXS_ERR_ARG;
  } else if (B.mode == MXS_ALLOC_BUDGET || B.mode == MXS_ALLOC_LAYER) {
    if (B.den <= 0 || B.num < 0 || B.fixed8 < 0) return MXS_ERR_ARG;
    if (B.mode == MXS_ALLOC_LAYER) {
      if (!layer_w) return MXS_ERR_ARG;
      for (int l = 0; l < n_layers; ++l)
        if (!(layer_w[l] >= 0.0) || !std::isfinite(layer_w[l])) return MXS_ERR_ARG;
    }
    __int128 cap, used;
    budget_base(n_layers, K, N, B, cap, used);
    if (used > cap) return MXS_ERR_BUDGET;           // before any launch
  } else {
    return MXS_ERR_ARG;
  }
  size_t need = 0;
  mxs_allocate_workspace_bytes(n_layers, K, &need);
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MXS_ERR_WORKSPACE;
  mxs_status st = check_device();
  if (st != MXS_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  std::vector<LayerWs> L(n_layers);
  uint8_t *p = reinterpret_cast<uint8_t *>(ws);
  for (int l = 0; l < n_layers; ++l) {
    L[l].rank = reinterpret_cast<int32_t *>(p);
    L[l].order = reinterpret_cast<int32_t *>(p + round_up(K[l] * 4, 256));
    L[l].gains = reinterpret_cast<double *>(p + 2 * round_up(K[l] * 4, 256));
    p += layer_ws_bytes(K[l]);
    launch_pdl(rank_kernel, dim3(static_cast<unsigned>((K[l] + kRankCols - 1) / kRankCols)), dim3(kRankThreads), 0, cs, s[l], K[l],
                                                                                                   L[l].rank);
    count_launch();
  }

  std::vector<int64_t> n8(n_layers, 0), n6(n_layers, 0);
  if (B.mode == MXS_ALLOC_FRACTIONS) {
    for (int l = 0; l < n_layers; ++l) {
      n8[l] = std::min(round_half_up_frac(B.p8_num, B.p8_den, K[l]), K[l]);
      n6[l] = std::min(round_half_up_frac(B.p6_num, B.p6_den, K[l]), K[l] - n8[l]);
    }
  } else if (B.mode == MXS_ALLOC_LAYER) {
    __int128 cap, used;
    budget_base(n_layers, K, N, B, cap, used);     // feasible: checked above
    for (int l = 0; l < n_layers; ++l) n8[l] = std::min(B.fixed8, K[l]);
    layer_rule(n_layers, K, N, layer_w, B, n8, cap, used, n6);
  } else {
    __int128 cap, used;
    budget_base(n_layers, K, N, B, cap, used);     // feasible: checked above
    for (int l = 0; l < n_layers; ++l) n8[l] = std::min(B.fixed8, K[l]);
    std::vector<std::vector<double>> gains(n_layers);
    if (n_layers > 1) {
      for (int l = 0; l < n_layers; ++l) {
        const int64_t ng = (K[l] - n8[l] + 31) / 32;
        gains[l].assign(static_cast<size_t>(std::max<int64_t>(ng, 1)), 0.0);
        if (ng > 0) {
          launch_pdl(order_kernel, dim3(static_cast<unsigned>((K[l] + 255) / 256)), dim3(256), 0, cs, L[l].rank, K[l], L[l].order);
          count_launch();
          launch_pdl(group_gain_kernel, dim3(static_cast<unsigned>((ng + 127) / 128)), dim3(128), 0, cs, s[l], L[l].order, K[l],
                                                                                    n8[l], ng, L[l].gains);
          count_launch();
          if (cudaMemcpyAsync(gains[l].data(), L[l].gains, static_cast<size_t>(ng) * 8,
                              cudaMemcpyDeviceToHost, cs) != cudaSuccess)
            return MXS_ERR_CUDA;
        }
      }
      if (cudaStreamSynchronize(cs) != cudaSuccess) return MXS_ERR_CUDA;
    }
    for (;;) {
      int best = -1;
      double best_gain = 0.0, best_cost = 0.0;
      for (int l = 0; l < n_layers; ++l) {
        const int64_t r0 = n8[l] + n6[l];
        if (r0 >= K[l]) continue;
        const int64_t cnt = std::min<int64_t>(32, K[l] - r0);
        const double w = layer_w ? layer_w[l] : 1.0;
        const double gain = n_layers > 1 ? w * gains[l][static_cast<size_t>(n6[l] / 32)] : 0.0;
        const double cost = static_cast<double>(2 * N[l] * cnt);
        if (best < 0 || gain * best_cost > best_gain * cost) {
          best = l;
          best_gain = gain;
          best_cost = cost;
        }
      }
      if (best < 0) break;
      const int64_t r0 = n8[best] + n6[best];
      const int64_t cnt = std::min<int64_t>(32, K[best] - r0);
      const __int128 add = static_cast<__int128>(B.den) * 2 * N[best] * cnt;
      if (used + add > cap) break;
      used += add;
      n6[best] += cnt;
    }
  }

  for (int l = 0; l < n_layers; ++l) {
    launch_pdl(perm_place_kernel, dim3(static_cast<unsigned>((K[l] + kPlaceCols - 1) / kPlaceCols)), dim3(kPlaceCols), 0,
               cs, L[l].rank, K[l], n8[l], n6[l], perm[l]);
    count_launch();
    counts[3 * l + 0] = n8[l];
    counts[3 * l + 1] = n6[l];
    counts[3 * l + 2] = K[l] - n8[l] - n6[l];
  }
  return cuda_status(cudaGetLastError());
}
