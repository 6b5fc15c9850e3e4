// mxs_attention.cu -- one decode step of grouped-query attention over the
// 4-bit MXINT K/V cache, reading the packed cache directly.
//
// MXSens (arXiv 2607.17733), technical summary §4: the W4A4KV4 setting keeps
// the K/V cache in 4-bit MXINT; the review's Validation section sets A4W4KV4
// against A4W4KV16.  The pages give no attention kernel; this one is written
// for sm_100a.
//
// Work split (split over tokens, then a combine): CTA (kv head g, split j)
// takes tokens [jC, jC + C) of kv head g for all rep = n_qh / n_kvh query
// heads of its group, so every cache byte is read once.  One thread issues
// four TMA tensor copies (K codes, K scales, V codes, V scales; 3-D maps over
// the [T][n_kvh][row] cache, box = one kv head x C tokens) on two barriers,
// so the scores run while V is still landing.  A second kernel merges the
// splits' (max, sum, partial output) triples.
//
// Decoding.  A 4-bit code x (two's complement nibble, value q) becomes the
// exact bf16 value q * 2^(e-2) of its block in one packed fma: the nibble
// with its sign bit flipped, placed in the mantissa of 128.0 (bits
// 0x4300 | (x ^ 8)), is the bf16 of 136 + q, and
// fma(136 + q, 2^(e-2), -136 * 2^(e-2)) rounds the exact value q 2^(e-2),
// which bf16 holds exactly (<= 3 significant bits), so it is that value.
// Two codes are decoded per instruction (bf16x2).
//
// Contractions on the tensor cores, mma.sync m16n8k16 bf16 with fp32
// accumulation:
//   scores S = deq(K) q^T: rows = 16 tokens, k = 16 head-dimension
//     positions, n = 8 query heads (the group, zero-padded); bf16 q times an
//     exact decoded key is exact in fp32, only the accumulation rounds;
//   output O^T = deq(V)^T P^T: rows = 16 head-dimension positions, k = 16
//     tokens, n = 8 heads; the softmax weights P (in [0, 1], unnormalised)
//     enter as a bf16 high part plus a bf16 remainder, two MMAs, so they
//     carry 16 significant bits.
// The contraction is 8 heads wide: tcgen05's smallest tile (M = 64) would
// leave most of the tensor core idle, and the step is bound by the cache's
// bytes, so the warp-level MMA is the right size here.  Both operands' order
// along k is free (a dot product), so each lane takes the codes that are
// contiguous in its registers and the other operand follows that order.
#include <cuda.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "mxs_internal.cuh"
#include "mxs_ptx.cuh"

namespace mxs {
namespace {

constexpr int kAttnD = 128;               // head dimension served
constexpr int kAttnWarps = 8;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kAttnMaxRep = 8;            // query heads per kv head: one n-tile of 8
constexpr int kAttnTargetCtas = 256;      // splits of 256 tokens: 16 token tiles, 2 per warp
constexpr int kAttnMinChunk = 64;
constexpr int kAttnMaxChunk = 256;        // a TMA box holds at most 256 rows
constexpr int kRowBytes = kAttnD / 2;     // packed codes of one cache row
constexpr int kScaleBox = 16;             // scale bytes copied per row (the row pitch's first 16)
constexpr long long kAttnWaitLimit = 2000000000LL;   // cycles (~1 s)

struct AttnArgs {
  const uint16_t *q;     // bf16 bits
  int64_t ldq;
  int32_t n_qh, n_kvh, rep, T, chunk, splits;
  float scale_log2;      // sm_scale * log2(e): scores kept in the base-2 domain
  float *part;           // [splits][n_qh][kAttnD + 2]: max (base 2), sum, partial output
  float *out;
  int64_t ldo;
};

struct AttnSmem {
  int32_t kc, ks, vc, vs, s, red, stat, bar, bytes;
};

__host__ __device__ inline AttnSmem attn_smem(int chunk) {
  AttnSmem p{};
  p.kc = 0;
  p.ks = p.kc + chunk * kRowBytes;
  p.vc = p.ks + chunk * kScaleBox;
  p.vs = p.vc + chunk * kRowBytes;
  p.s = p.vs + chunk * kScaleBox;
  p.red = p.s + kAttnMaxRep * chunk * 4;
  p.stat = p.red + kAttnWarps * kAttnMaxRep * kAttnD * 4;     // per head: max, sum
  p.bar = p.stat + 2 * kAttnMaxRep * 4;
  p.bytes = p.bar + 16 + 128;                                  // + slack to align the base to 128 bytes
  return p;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t fma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// bf16 bits of the block step 2^(e-2) for E8M0 byte b = e + 127 (subnormal
// for b <= 2).
__device__ __forceinline__ uint32_t step_bits(uint32_t b) { return b >= 3u ? (b - 2u) << 7 : 1u << (b + 4u); }
// bf16 bits of -136 * 2^(e-2) = -1.0625 * 2^(b-122) (b <= 249).
__device__ __forceinline__ uint32_t neg136_bits(uint32_t b) { return 0x8000u | ((b + 5u) << 7) | 8u; }
// Two codes -- the low nibbles of the two 16-bit halves of x -- decoded to
// bf16 with the steps / offsets in s2 / c2 (one pair per half).
__device__ __forceinline__ uint32_t decode2(uint32_t x, uint32_t s2, uint32_t c2) {
  return fma2((x & 0x000F000Fu) ^ 0x43084308u, s2, c2);
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// bf16x2 of (lo, hi), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(ptx::smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(ptx::smem_addr(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

}  // namespace

// CTA (g, j): kv head g = blockIdx.x / splits, split j = blockIdx.x % splits.
__global__ void __launch_bounds__(kAttnThreads) attn_split_kernel(const __grid_constant__ CUtensorMap mKc,
                                                                  const __grid_constant__ CUtensorMap mKs,
                                                                  const __grid_constant__ CUtensorMap mVc,
                                                                  const __grid_constant__ CUtensorMap mVs,
                                                                  AttnArgs a, int *status) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  // TMA destinations want 128-byte alignment
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int g = blockIdx.x / a.splits, sp = blockIdx.x - g * a.splits;
  const int t0 = sp * a.chunk;
  const int nt = min(a.chunk, a.T - t0);              // >= 1 (the host sizes the splits)
  const int ntiles = (nt + 15) >> 4;
  const AttnSmem L = attn_smem(a.chunk);
  uint8_t *kc = smem + L.kc, *ks = smem + L.ks, *vc = smem + L.vc, *vs = smem + L.vs;
  float *S = reinterpret_cast<float *>(smem + L.s);
  float *red = reinterpret_cast<float *>(smem + L.red);
  float *head_max = reinterpret_cast<float *>(smem + L.stat), *head_sum = head_max + kAttnMaxRep;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L.bar);

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar[0], 1);
    ptx::mbar_init(&bar[1], 1);
    ptx::fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(&mKc) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&mVc) : "memory");
  }
  __syncthreads();
  pdl_wait();                                          // the cache and q come from earlier kernels
  if (threadIdx.x == 0) {
    const uint32_t bytes = static_cast<uint32_t>(a.chunk) * (kRowBytes + kScaleBox);
    ptx::mbar_arrive_expect_tx(&bar[0], bytes);
    tma_load_3d(kc, &mKc, &bar[0], 0, g, t0);
    tma_load_3d(ks, &mKs, &bar[0], 0, g, t0);
    ptx::mbar_arrive_expect_tx(&bar[1], bytes);
    tma_load_3d(vc, &mVc, &bar[1], 0, g, t0);
    tma_load_3d(vs, &mVs, &bar[1], 0, g, t0);
  }

  // q as the scores' B operand: head n = gid of the group, k = the lane's
  // 32 head-dimension positions 32 tig .. 32 tig + 31 in the order the key
  // codes take them (step s: positions 8(s/2) + 2(s%2) + {0, 4} for b0 and
  // + {1, 5} for b1).  Rows past the group are zero.
  uint32_t qb[8][2];
  {
    uint32_t w[16];
    if (gid < a.rep) {
      const uint4 *src = reinterpret_cast<const uint4 *>(a.q + static_cast<int64_t>(g * a.rep + gid) * a.ldq + 32 * tig);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = __ldg(src + i);
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i] = 0u;
    }
    // bf16 at offset o is half (o & 1) of w[o >> 1]; pair(o1, o2) puts o1 low, o2 high
#pragma unroll
    for (int s = 0; s < 8; ++s) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int o1 = 8 * (s >> 1) + 2 * (s & 1) + h, o2 = o1 + 4;
        const uint32_t sel = ((o1 & 1) ? 0x0032u : 0x0010u) | ((o2 & 1) ? 0x7600u : 0x5400u);
        qb[s][h] = prmt(w[o1 >> 1], w[o2 >> 1], sel);
      }
    }
  }

  // ---- scores: warp w takes 16-token tiles w, w + 8, ...
  auto landed = [&](int c) -> bool {
    const bool ok = ptx::mbar_wait_cycles(&bar[c], 0, kAttnWaitLimit);
    if (!__syncthreads_or(!ok)) return true;
    if (threadIdx.x == 0) {
      atomicExch(status, static_cast<int>(MXS_ERR_TIMEOUT));
      if (c == 0) ptx::mbar_wait_cycles(&bar[1], 0, kAttnWaitLimit);   // leave no copy in flight
    }
    return false;
  };
  if (!landed(0)) return;
  for (int kt = warp; kt < ntiles; kt += kAttnWarps) {
    const int r0 = 16 * kt + gid, r1 = r0 + 8;
    const uint4 k0 = *reinterpret_cast<const uint4 *>(kc + r0 * kRowBytes + 16 * tig);
    const uint4 k1 = *reinterpret_cast<const uint4 *>(kc + r1 * kRowBytes + 16 * tig);
    const uint32_t e0 = ks[r0 * kScaleBox + tig], e1 = ks[r1 * kScaleBox + tig];
    const uint32_t s0 = step_bits(e0) * 0x10001u, c0 = neg136_bits(e0) * 0x10001u;
    const uint32_t s1 = step_bits(e1) * 0x10001u, c1 = neg136_bits(e1) * 0x10001u;
    const uint32_t kw0[4] = {k0.x, k0.y, k0.z, k0.w}, kw1[4] = {k1.x, k1.y, k1.z, k1.w};
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int j = s >> 1, i = 2 * (s & 1);
      uint32_t fa[4];
      fa[0] = decode2(kw0[j] >> (4 * i), s0, c0);          // token r0: codes 8j+i, 8j+i+4
      fa[1] = decode2(kw1[j] >> (4 * i), s1, c1);          // token r1
      fa[2] = decode2(kw0[j] >> (4 * i + 4), s0, c0);      // codes 8j+i+1, 8j+i+5
      fa[3] = decode2(kw1[j] >> (4 * i + 4), s1, c1);
      mma16816(acc, fa, qb[s][0], qb[s][1]);
    }
    const float ninf = -INFINITY;
    S[(2 * tig) * a.chunk + r0] = r0 < nt ? acc[0] * a.scale_log2 : ninf;
    S[(2 * tig + 1) * a.chunk + r0] = r0 < nt ? acc[1] * a.scale_log2 : ninf;
    S[(2 * tig) * a.chunk + r1] = r1 < nt ? acc[2] * a.scale_log2 : ninf;
    S[(2 * tig + 1) * a.chunk + r1] = r1 < nt ? acc[3] * a.scale_log2 : ninf;
  }
  __syncthreads();

  // ---- softmax over the split, warp h for head h: max, then weights 2^(s - max)
  {
    float *row = S + warp * a.chunk;
    const int nfill = ntiles * 16;
    if (warp < a.rep) {
      float m = -INFINITY;
      for (int t = lane; t < nt; t += 32) m = fmaxf(m, row[t]);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float sum = 0.f;
      for (int t = lane; t < nfill; t += 32) {
        const float p = t < nt ? exp2f(row[t] - m) : 0.f;
        row[t] = p;
        sum += p;
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        head_max[warp] = m;
        head_sum[warp] = sum;
      }
    } else {
      for (int t = lane; t < nfill; t += 32) row[t] = 0.f;
    }
  }
  if (!landed(1)) return;                              // (its barrier also publishes the weights)

  // ---- output: O^T tile m holds head-dimension rows 16 gid + m (codes of
  // word 2 gid) and 16 gid + 8 + m (word 2 gid + 1); the lane's k positions
  // are tokens tig, tig + 4 (b0 / a0, a1) and tig + 8, tig + 12 (b1 / a2, a3)
  float o[8][4];
#pragma unroll
  for (int m = 0; m < 8; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[m][i] = 0.f;
  const float *prow = S + gid * a.chunk;
  for (int kt = warp; kt < ntiles; kt += kAttnWarps) {
    const int ta = 16 * kt + tig, tb = ta + 4, tc = ta + 8, td = ta + 12;
    const uint2 va = *reinterpret_cast<const uint2 *>(vc + ta * kRowBytes + 8 * gid);
    const uint2 vb = *reinterpret_cast<const uint2 *>(vc + tb * kRowBytes + 8 * gid);
    const uint2 vcc = *reinterpret_cast<const uint2 *>(vc + tc * kRowBytes + 8 * gid);
    const uint2 vd = *reinterpret_cast<const uint2 *>(vc + td * kRowBytes + 8 * gid);
    const int blk = gid >> 1;                          // positions 16 gid .. 16 gid + 15: one block
    const uint32_t ea = vs[ta * kScaleBox + blk], eb = vs[tb * kScaleBox + blk];
    const uint32_t ec = vs[tc * kScaleBox + blk], ed = vs[td * kScaleBox + blk];
    const uint32_t sab = step_bits(ea) | (step_bits(eb) << 16), cab = neg136_bits(ea) | (neg136_bits(eb) << 16);
    const uint32_t scd = step_bits(ec) | (step_bits(ed) << 16), ccd = neg136_bits(ec) | (neg136_bits(ed) << 16);
    // P as the B operand (head gid), high bf16 part and remainder
    const float pa = prow[ta], pb = prow[tb], pc = prow[tc], pd = prow[td];
    const uint32_t hi0 = pack_bf16x2(pa, pb), hi1 = pack_bf16x2(pc, pd);
    const uint32_t lo0 = pack_bf16x2(pa - __uint_as_float(hi0 << 16), pb - __uint_as_float(hi0 & 0xFFFF0000u));
    const uint32_t lo1 = pack_bf16x2(pc - __uint_as_float(hi1 << 16), pd - __uint_as_float(hi1 & 0xFFFF0000u));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // byte k of each token's word: codes 2k (low nibble) and 2k + 1 of the word
      const uint32_t sel = static_cast<uint32_t>(k) | (static_cast<uint32_t>(4 + k) << 8);
      const uint32_t x0 = prmt(va.x, vb.x, sel), x1 = prmt(va.y, vb.y, sel);
      const uint32_t x2 = prmt(vcc.x, vd.x, sel), x3 = prmt(vcc.y, vd.y, sel);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int m = 2 * k + h;
        uint32_t fa[4];
        fa[0] = decode2(x0 >> (4 * h), sab, cab);
        fa[1] = decode2(x1 >> (4 * h), sab, cab);
        fa[2] = decode2(x2 >> (4 * h), scd, ccd);
        fa[3] = decode2(x3 >> (4 * h), scd, ccd);
        mma16816(o[m], fa, hi0, hi1);
        mma16816(o[m], fa, lo0, lo1);
      }
    }
  }
  // the warps' partial outputs, added in warp order
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    float *rw = red + warp * (kAttnMaxRep * kAttnD);
    const int d0 = 16 * gid + m, d1 = d0 + 8;
    rw[(2 * tig) * kAttnD + d0] = o[m][0];
    rw[(2 * tig + 1) * kAttnD + d0] = o[m][1];
    rw[(2 * tig) * kAttnD + d1] = o[m][2];
    rw[(2 * tig + 1) * kAttnD + d1] = o[m][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < a.rep * kAttnD; i += kAttnThreads) {
    const int h = i / kAttnD, d = i - h * kAttnD;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) sum += red[(w * kAttnMaxRep + h) * kAttnD + d];
    float *dst = a.part + (static_cast<int64_t>(sp) * a.n_qh + g * a.rep + h) * (kAttnD + 2);
    dst[2 + d] = sum;
    if (d == 0) {
      dst[0] = head_max[h];
      dst[1] = head_sum[h];
    }
  }
}

// One CTA per query head.  The splits' weights 2^(m_j - M) rescale their
// sums and partial outputs; thread (group r, position d) adds the splits
// j = r, r + 4, ... for position d with several loads in flight, and the
// four groups are added in group order (the result does not depend on the
// launch).
constexpr int kCombGroups = 4;
constexpr int kCombThreads = kCombGroups * kAttnD;

__global__ void __launch_bounds__(kCombThreads) attn_combine_kernel(AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[kCombGroups][kAttnD];
  __shared__ float wred[kCombThreads / 32];
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t stride = static_cast<int64_t>(a.n_qh) * (kAttnD + 2);
  const float *p = a.part + static_cast<int64_t>(h) * (kAttnD + 2);
  // M = max_j m_j
  float m = -INFINITY;
  for (int j = tid; j < a.splits; j += kCombThreads) m = fmaxf(m, p[j * stride]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) wred[warp] = m;
  __syncthreads();
  float M = wred[0];
#pragma unroll
  for (int w = 1; w < kCombThreads / 32; ++w) M = fmaxf(M, wred[w]);
  __syncthreads();
  // the denominator sum_j 2^(m_j - M) l_j, in split order (one warp)
  if (warp == 0) {
    float den = 0.f;
    for (int j0 = 0; j0 < a.splits; j0 += 32) {
      const int j = j0 + lane;
      float v = j < a.splits ? exp2f(p[j * stride] - M) * p[j * stride + 1] : 0.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;                        // prefix sums: lane 31 holds the 32-split sum
      }
      den += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) wred[0] = den;
  }
  const int r = tid / kAttnD, d = tid - r * kAttnD;
  float num = 0.f;
#pragma unroll 4
  for (int j = r; j < a.splits; j += kCombGroups) {
    const float *pj = p + j * stride;
    num = fmaf(exp2f(pj[0] - M), pj[2 + d], num);
  }
  red[r][d] = num;
  __syncthreads();
  if (r == 0) {
    float sum = red[0][d];
#pragma unroll
    for (int g = 1; g < kCombGroups; ++g) sum += red[g][d];
    a.out[static_cast<int64_t>(h) * a.ldo + d] = sum / wred[0];
  }
}

namespace {

// Tokens per split: about two CTAs per SM over all kv heads, a multiple of
// the 16-token tile, within one TMA box.
int attn_chunk(int64_t T, int64_t n_kvh) {
  int64_t c = (T * n_kvh + kAttnTargetCtas - 1) / kAttnTargetCtas;
  c = std::max<int64_t>(kAttnMinChunk, std::min<int64_t>(kAttnMaxChunk, round_up(c, 16)));
  return static_cast<int>(std::min<int64_t>(c, round_up(T, 16)));
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D byte map over a cache of T x n_kvh rows at `pitch` bytes: x = the
// first `cols` bytes of a row, y = kv head, z = token; box cols x 1 x chunk.
bool cache_map(CUtensorMap *m, const uint8_t *base, int64_t cols, int64_t pitch, int64_t n_kvh, int64_t T,
               int box_cols, int chunk) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(n_kvh),
                              static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(pitch), static_cast<cuuint64_t>(pitch * n_kvh)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), 1u, static_cast<cuuint32_t>(chunk)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool kv_layout_ok(const mxs_mxtensor *t, int64_t rows) {
  const mxs_layout &l = t->lay;
  return t->rows == rows && l.perm == nullptr && l.K == kAttnD && l.seg[0].k_real == 0 && l.seg[1].k_real == 0 &&
         l.seg[2].k_real == kAttnD;
}

}  // namespace
}  // namespace mxs

using namespace mxs;

extern "C" mxs_status mxs_attn_decode_workspace_bytes(int64_t T, int64_t n_qh, int64_t n_kvh, int64_t d,
                                                      size_t *bytes) {
  if (!bytes || T < 1 || n_qh < 1 || n_kvh < 1) return MXS_ERR_ARG;
  if (d != kAttnD || n_qh % n_kvh || n_qh / n_kvh > kAttnMaxRep || T > INT32_MAX / 2 || n_kvh > 65535)
    return MXS_ERR_SHAPE;
  const int64_t splits = (T + attn_chunk(T, n_kvh) - 1) / attn_chunk(T, n_kvh);
  *bytes = static_cast<size_t>(splits * n_qh * (kAttnD + 2) * 4);
  return MXS_OK;
}

extern "C" mxs_status mxs_attn_decode(const void *q, int64_t n_qh, int64_t ldq, const mxs_mxtensor *K,
                                      const mxs_mxtensor *V, int64_t T, int64_t n_kvh, float sm_scale, float *out,
                                      int64_t ldo, void *ws, size_t ws_bytes, void *stream) {
  if (!q || !K || !V || !out) return MXS_ERR_ARG;
  size_t need = 0;
  mxs_status st = mxs_attn_decode_workspace_bytes(T, n_qh, n_kvh, K->lay.K, &need);
  if (st != MXS_OK) return st;
  if (!std::isfinite(sm_scale)) return MXS_ERR_ARG;
  if ((st = check_mxtensor(K)) != MXS_OK || (st = check_mxtensor(V)) != MXS_OK) return st;
  if (!kv_layout_ok(K, T * n_kvh) || !kv_layout_ok(V, T * n_kvh)) return MXS_ERR_SHAPE;
  if (ldq < kAttnD || ldo < kAttnD) return MXS_ERR_SHAPE;
  if (!aligned16(q) || (ldq * 2) % 16) return MXS_ERR_ALIGN;
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MXS_ERR_WORKSPACE;
  if ((st = check_device()) != MXS_OK) return st;

  AttnArgs a{};
  a.q = static_cast<const uint16_t *>(q);
  a.ldq = ldq;
  a.n_qh = static_cast<int32_t>(n_qh);
  a.n_kvh = static_cast<int32_t>(n_kvh);
  a.rep = static_cast<int32_t>(n_qh / n_kvh);
  a.T = static_cast<int32_t>(T);
  a.chunk = attn_chunk(T, n_kvh);
  a.splits = static_cast<int32_t>((T + a.chunk - 1) / a.chunk);
  a.scale_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634);   // log2(e)
  a.part = static_cast<float *>(ws);
  a.out = out;
  a.ldo = ldo;
  if (static_cast<int64_t>(a.splits) * n_kvh > INT32_MAX) return MXS_ERR_SHAPE;

  CUtensorMap mKc{}, mKs{}, mVc{}, mVs{};
  const int seg = 2;   // the 4-bit segment
  if (!cache_map(&mKc, K->codes[seg], kRowBytes, K->code_pitch[seg], n_kvh, T, kRowBytes, a.chunk) ||
      !cache_map(&mKs, K->scales[seg], K->scale_pitch[seg], K->scale_pitch[seg], n_kvh, T, kScaleBox, a.chunk) ||
      !cache_map(&mVc, V->codes[seg], kRowBytes, V->code_pitch[seg], n_kvh, T, kRowBytes, a.chunk) ||
      !cache_map(&mVs, V->scales[seg], V->scale_pitch[seg], V->scale_pitch[seg], n_kvh, T, kScaleBox, a.chunk))
    return MXS_ERR_CUDA;
  int *status = device_status_word();
  if (!status) return MXS_ERR_CUDA;
  const int smem = attn_smem(a.chunk).bytes;
  if (!ensure_smem(attn_split_kernel, smem)) return MXS_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  launch_pdl(attn_split_kernel, dim3(static_cast<unsigned>(a.splits * n_kvh)), dim3(kAttnThreads),
             static_cast<size_t>(smem), cs, mKc, mKs, mVc, mVs, a, status);
  launch_pdl(attn_combine_kernel, dim3(static_cast<unsigned>(n_qh)), dim3(kCombThreads), 0, cs, a);
  count_launch(2);
  return cuda_status(cudaGetLastError());
}
