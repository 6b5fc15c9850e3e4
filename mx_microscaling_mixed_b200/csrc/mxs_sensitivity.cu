// mxs_sensitivity.cu -- column sensitivity s_j = H_jj * E_j of one layer.
//
// MXSens (arXiv 2607.17733), technical summary §2.1: column-wise sensitivity
// from the diagonal of the empirical Hessian H = X^T X; columns carrying large
// outliers have large H_jj.  Fixed reading: H_jj = (2/T) sum_t X_tj^2 and
// E_j = sum_i (W_ij - Q4(W)_ij)^2 with Q4 the 4-bit MXINT code of each W row
// in blocks of 32 original columns.
//
// Rounding order (pinned so that every launch shape gives the same bits):
// rows are cut into chunks of 64; a chunk is summed from zero in row order in
// fp64; chunk sums are then added in chunk order.  Each term is the square
// of an fp32/bf16 value or of the exact difference W - Q4(W); both have at
// most 26 significant bits, so the square is exact in fp64 and one fused
// multiply-add adds it with a single rounding, the same bits as a rounded
// product followed by a rounded add.  The remaining operations use explicit
// round-to-nearest intrinsics, so no contraction can change the result.
//
// Two launches.  (1) Chunk partials: one CTA (one warp) per 64-row chunk x
// 256-column tile of X or of W; one thread streams the chunk through two
// 8-row shared-memory buffers by TMA (zero fill past the matrix edge, which
// adds exact zeros and leaves block maxima alone) and each lane owns 8
// consecutive columns, walking the chunk's rows in order; on the W side the
// 4 lanes that own one 32-column block share its maximum through two
// xor-shuffles.  The small buffers let many CTAs share an SM, so loads stay
// in flight while others compute.  Rows or pitches that a TMA map cannot
// describe (unaligned base or pitch) take a register-streaming variant with
// the same arithmetic.  (2) A per-column pass that stages the chunk
// partials of 16 columns in shared memory (all of a thread's loads in flight
// together), adds them in chunk order and forms H, E and s.
#include <algorithm>
#include <mutex>

#include "mxs_internal.cuh"
#include "mxs_ptx.cuh"

namespace mxs {

constexpr int kSumChunk = 64;
constexpr int kSensThreads = 256;
constexpr int kColsPerThread = 4;

struct SensArgs {
  const void *X;
  const void *W;
  int64_t T, N, K, ldx, ldw;
  int32_t nchunk_x, nchunk_w;
  double *part;        // (nchunk_x + nchunk_w) x K
};

template <bool F32, bool VEC>
__device__ __forceinline__ void load4(const void *base, int64_t row_off, int64_t c0, int64_t K,
                                      float (&v)[kColsPerThread]) {
  if (VEC && c0 + kColsPerThread <= K) {
    if constexpr (F32) {
      const float4 a = __ldg(reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + row_off + c0));
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else {
      const uint2 a = __ldg(reinterpret_cast<const uint2 *>(reinterpret_cast<const unsigned short *>(base) + row_off + c0));
      v[0] = __uint_as_float(a.x << 16);
      v[1] = __uint_as_float(a.x & 0xFFFF0000u);
      v[2] = __uint_as_float(a.y << 16);
      v[3] = __uint_as_float(a.y & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kColsPerThread; ++i) {
      const int64_t c = c0 + i;
      float x = 0.f;
      if (c < K) {
        if constexpr (F32) x = __ldg(reinterpret_cast<const float *>(base) + row_off + c);
        else x = bf16_bits_to_float(__ldg(reinterpret_cast<const unsigned short *>(base) + row_off + c));
      }
      v[i] = x;
    }
  }
}

__device__ __forceinline__ double pow2d(int k) {
  return __longlong_as_double(static_cast<long long>(k + 1023) << 52);
}

constexpr int kRowBatch = 8;   // rows loaded ahead per thread

// acc + d^2 rounded once.  Every d here has at most 26 significant bits and
// an exponent within fp32's range widened by a few bits, so d^2 is exact in
// fp64 and the fused form equals the product rounded and then added.
__device__ __forceinline__ double add_square(double acc, double d) { return __fma_rn(d, d, acc); }

// w - Q4(w) in fp64, Q4 the 4-bit code under the block exponent:
// sc = 2^(2-e) (a normal float), step = 2^(e-2).  The code comes from
// fma(w, sc, 1.5*2^23) (round half to even), clamped on its bit pattern; the
// same pattern minus 1.5*2^23 is the code as a float.  For bf16 w the
// difference w - q*step has <= 9 significant bits on the bf16 grid and is
// exact in fp32; for fp32 w it is formed in fp64.
template <bool F32>
__device__ __forceinline__ double q4_err(float w, float sc, float step) {
  uint32_t x = __float_as_uint(fmaf(w, sc, 12582912.0f));
  x = min(max(x, 0x4B400000u - 7u), 0x4B400000u + 7u);
  const float qv = __fmul_rn(__uint_as_float(x) - 12582912.0f, step);     // exact
  if constexpr (F32) return __dsub_rn(static_cast<double>(w), static_cast<double>(qv));
  else return static_cast<double>(__fsub_rn(w, qv));
}

// The same difference for a block whose maximum is below 2^-125, where
// 2^(2-e) is not a normal float: the code is found on the input pre-scaled
// by 2^64 and the difference is formed in fp64.
__device__ __forceinline__ double q4_err_tiny(float w, int e) {
  const float sc = __uint_as_float(static_cast<uint32_t>(2 - e - 64 + 127) << 23);
  uint32_t x = __float_as_uint(fmaf(w * 18446744073709551616.0f, sc, 12582912.0f));
  x = min(max(x, 0x4B400000u - 7u), 0x4B400000u + 7u);
  const double q = static_cast<double>(__uint_as_float(x) - 12582912.0f);
  return __dsub_rn(static_cast<double>(w), __dmul_rn(q, pow2d(e - 2)));
}

template <bool XF32, bool WF32, bool XVEC, bool WVEC>
__global__ void __launch_bounds__(kSensThreads) sens_partial_kernel(SensArgs a) {
  pdl_wait();
  pdl_trigger();
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * kSensThreads + threadIdx.x;
  const int64_t c0 = gtid * kColsPerThread;
  double acc[kColsPerThread];
#pragma unroll
  for (int i = 0; i < kColsPerThread; ++i) acc[i] = 0.0;
  const int chunk = blockIdx.y;
  if (chunk < a.nchunk_x) {
    if (c0 >= a.K) return;                      // no cross-lane work on this side
    const int64_t r0 = static_cast<int64_t>(chunk) * kSumChunk;
    const int64_t r1 = min(r0 + kSumChunk, a.T);
    for (int64_t t = r0; t < r1; t += kRowBatch) {
      float v[kRowBatch][kColsPerThread];
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        if (t + u < r1) load4<XF32, XVEC>(a.X, (t + u) * a.ldx, c0, a.K, v[u]);
      }
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        if (t + u < r1) {
#pragma unroll
          for (int i = 0; i < kColsPerThread; ++i) acc[i] = add_square(acc[i], static_cast<double>(v[u][i]));
        }
      }
    }
  } else {
    // All lanes stay to the end: the block maximum needs the 8 owner lanes.
    const int wchunk = chunk - a.nchunk_x;
    const int64_t r0 = static_cast<int64_t>(wchunk) * kSumChunk;
    const int64_t r1 = min(r0 + kSumChunk, a.N);
    for (int64_t t = r0; t < r1; t += kRowBatch) {
      float v[kRowBatch][kColsPerThread];
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        if (t + u < r1) load4<WF32, WVEC>(a.W, (t + u) * a.ldw, c0, a.K, v[u]);
      }
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        if (t + u < r1) {                       // uniform across the warp
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < kColsPerThread; ++i) amax = fmaxf(amax, fabsf(v[u][i]));
          uint32_t ab = __float_as_uint(amax);
          ab = max(ab, __shfl_xor_sync(0xffffffffu, ab, 1));   // 8 lanes own one 32-column block
          ab = max(ab, __shfl_xor_sync(0xffffffffu, ab, 2));
          ab = max(ab, __shfl_xor_sync(0xffffffffu, ab, 4));
          const int ef = static_cast<int>(ab >> 23);
          const int e = ef == 0 ? -127 : ef - 127;
          if (e >= -125) {
            const float sc = __uint_as_float(static_cast<uint32_t>(2 - e + 127) << 23);
            const float step = pow2f(e - 2);
#pragma unroll
            for (int i = 0; i < kColsPerThread; ++i) acc[i] = add_square(acc[i], q4_err<WF32>(v[u][i], sc, step));
          } else {
#pragma unroll
            for (int i = 0; i < kColsPerThread; ++i) acc[i] = add_square(acc[i], q4_err_tiny(v[u][i], e));
          }
        }
      }
    }
    if (c0 >= a.K) return;
  }
  double *out = a.part + static_cast<int64_t>(chunk) * a.K + c0;
#pragma unroll
  for (int i = 0; i < kColsPerThread; ++i)
    if (c0 + i < a.K) out[i] = acc[i];
}

constexpr int kTileCols = 256;                        // columns per tile
constexpr int kTileCPT = 8;                           // columns per thread in the tile kernel
constexpr int kTileThreads = kTileCols / kTileCPT;
constexpr long long kTileWaitLimit = 2000000000LL;    // cycles (~1 s)

// Row r of a staged fp32 tile: this thread's 8 values.
__device__ __forceinline__ void lds_row_f32(const uint8_t *tile, int r, int cl, float (&v)[kTileCPT]) {
  const float4 *p = reinterpret_cast<const float4 *>(tile + (static_cast<int64_t>(r) * kTileCols + cl) * 4);
  const float4 a = p[0], b = p[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Row r of a staged bf16 tile: this thread's 8 values as 4 packed words.
__device__ __forceinline__ void lds_row_bf16(const uint8_t *tile, int r, int cl, uint32_t (&p)[kTileCPT / 2]) {
  const uint4 a = *reinterpret_cast<const uint4 *>(tile + (static_cast<int64_t>(r) * kTileCols + cl) * 2);
  p[0] = a.x; p[1] = a.y; p[2] = a.z; p[3] = a.w;
}

__device__ __forceinline__ void unpack_bf16(const uint32_t (&p)[kTileCPT / 2], float (&v)[kTileCPT]) {
#pragma unroll
  for (int j = 0; j < kTileCPT / 2; ++j) {
    v[2 * j] = __uint_as_float(p[j] << 16);
    v[2 * j + 1] = __uint_as_float(p[j] & 0xFFFF0000u);
  }
}

// max(|a|, |b|) per bf16 half (the sign of the result is dropped by the caller).
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// w - Q4(w) for a bf16 w in the common case (block exponent e >= -125):
// the code comes from fma(w, 2^(2-e), 1.5*2^23) clamped on its bit pattern;
// w - q*2^(e-2) has <= 9 significant bits, so the fma that forms it is exact.
__device__ __forceinline__ double q4_err_bf16(float w, float sc, float step) {
  uint32_t x = __float_as_uint(fmaf(w, sc, 12582912.0f));
  x = min(max(x, 0x4B400000u - 7u), 0x4B400000u + 7u);
  return static_cast<double>(fmaf(-(__uint_as_float(x) - 12582912.0f), step, w));
}

// One row of this thread's W values: adds (w - Q4(w))^2 to acc under the
// 32-column block's exponent e (the block spans the 4 lanes that share it;
// `ab` is this lane's largest magnitude as fp32 bits).
template <bool F32>
__device__ __forceinline__ void w_row_terms(const float (&v)[kTileCPT], uint32_t ab, double (&acc)[kTileCPT]) {
#pragma unroll
  for (int m = 1; m < 32 / kTileCPT; m <<= 1) ab = max(ab, __shfl_xor_sync(0xffffffffu, ab, m));
  const int ef = static_cast<int>(ab >> 23);
  const int e = ef == 0 ? -127 : ef - 127;
  if (e >= -125) {
    const float sc = __uint_as_float(static_cast<uint32_t>(2 - e + 127) << 23);
    const float step = pow2f(e - 2);
#pragma unroll
    for (int i = 0; i < kTileCPT; ++i) {
      if constexpr (F32) acc[i] = add_square(acc[i], q4_err<true>(v[i], sc, step));
      else acc[i] = add_square(acc[i], q4_err_bf16(v[i], sc, step));
    }
  } else {
#pragma unroll
    for (int i = 0; i < kTileCPT; ++i) acc[i] = add_square(acc[i], q4_err_tiny(v[i], e));
  }
}

// Tiles in launch order: all X tiles (chunk-major), then all W tiles.  A
// tile (one 64-row chunk x 256 columns) streams through kSubBufs shared-memory
// buffers of kSubRows rows, so the next rows load while these are summed
// and a CTA needs little shared memory: many CTAs share an SM.
constexpr int kSubRows = 8;
constexpr int kSubBufs = 2;       // sub-tiles in flight per CTA

template <bool XF32, bool WF32>
__global__ void __launch_bounds__(kTileThreads)
    sens_tile_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW, SensArgs a,
                     int32_t ctiles, int *status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t tile[];
  __shared__ __align__(8) uint64_t bar[kSubBufs];
  const int nx = a.nchunk_x * ctiles;
  const bool is_x = static_cast<int>(blockIdx.x) < nx;
  const int t = is_x ? blockIdx.x : blockIdx.x - nx;
  const int chunk = t / ctiles, ct = t - chunk * ctiles;
  const bool f32 = is_x ? XF32 : WF32;
  const CUtensorMap *map = is_x ? &mapX : &mapW;
  const uint32_t sub_bytes = static_cast<uint32_t>(kSubRows * kTileCols * (f32 ? 4 : 2));
  const uint32_t buf_bytes = static_cast<uint32_t>(kSubRows * kTileCols * ((XF32 || WF32) ? 4 : 2));
  const int64_t r0 = static_cast<int64_t>(chunk) * kSumChunk;
  const int rows = static_cast<int>(min(static_cast<int64_t>(kSumChunk), (is_x ? a.T : a.N) - r0));
  const int nsub = (rows + kSubRows - 1) / kSubRows;
  if (threadIdx.x == 0) {
    for (int b = 0; b < kSubBufs; ++b) ptx::mbar_init(&bar[b], 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int b = 0; b < kSubBufs && b < nsub; ++b) {
      ptx::mbar_arrive_expect_tx(&bar[b], sub_bytes);
      ptx::tma_load_2d(tile + b * buf_bytes, map, &bar[b], ct * kTileCols, static_cast<int>(r0) + b * kSubRows);
    }
  }
  const int cl = threadIdx.x * kTileCPT;
  const int64_t c0 = static_cast<int64_t>(ct) * kTileCols + cl;
  double acc[kTileCPT];
#pragma unroll
  for (int i = 0; i < kTileCPT; ++i) acc[i] = 0.0;
  for (int sb = 0; sb < nsub; ++sb) {
    const int buf = sb % kSubBufs;
    if (!ptx::mbar_wait_cycles(&bar[buf], (sb / kSubBufs) & 1, kTileWaitLimit)) {
      // the other buffers' loads, if any, land before the CTA exits
      if (threadIdx.x == 0) {
        atomicExch(status, static_cast<int>(MXS_ERR_TIMEOUT));
        for (int b = sb + 1; b < sb + kSubBufs && b < nsub; ++b)
          ptx::mbar_wait_cycles(&bar[b % kSubBufs], (b / kSubBufs) & 1, kTileWaitLimit);
      }
      return;
    }
    const uint8_t *sub = tile + buf * buf_bytes;
    const int rr = min(kSubRows, rows - sb * kSubRows);
    if (is_x) {
#pragma unroll 8
      for (int r = 0; r < rr; ++r) {
        float v[kTileCPT];
        if constexpr (XF32) {
          lds_row_f32(sub, r, cl, v);
        } else {
          uint32_t p[kTileCPT / 2];
          lds_row_bf16(sub, r, cl, p);
          unpack_bf16(p, v);
        }
#pragma unroll
        for (int i = 0; i < kTileCPT; ++i) acc[i] = add_square(acc[i], static_cast<double>(v[i]));
      }
    } else {
#pragma unroll 4
      for (int r = 0; r < rr; ++r) {     // rr is uniform over the CTA
        float v[kTileCPT];
        uint32_t ab;
        if constexpr (WF32) {
          lds_row_f32(sub, r, cl, v);
          ab = 0;
#pragma unroll
          for (int i = 0; i < kTileCPT; ++i) ab = max(ab, __float_as_uint(v[i]) & 0x7FFFFFFFu);
        } else {
          uint32_t p[kTileCPT / 2];
          lds_row_bf16(sub, r, cl, p);
          unpack_bf16(p, v);
          const uint32_t m = maxabs_bf16x2(maxabs_bf16x2(p[0], p[1]), maxabs_bf16x2(p[2], p[3])) & 0x7FFF7FFFu;
          ab = max(m << 16, m & 0xFFFF0000u);      // the larger half, as fp32 bits
        }
        w_row_terms<WF32>(v, ab, acc);
      }
    }
    // the warp is done with this buffer: it takes the rows kSubBufs sub-tiles on
    __syncthreads();
    if (threadIdx.x == 0 && sb + kSubBufs < nsub) {
      ptx::mbar_arrive_expect_tx(&bar[buf], sub_bytes);
      ptx::tma_load_2d(tile + buf * buf_bytes, map, &bar[buf], ct * kTileCols,
                       static_cast<int>(r0) + (sb + kSubBufs) * kSubRows);
    }
  }
  double *out = a.part + static_cast<int64_t>(is_x ? chunk : a.nchunk_x + chunk) * a.K + c0;
#pragma unroll
  for (int i = 0; i < kTileCPT; ++i)
    if (c0 + i < a.K) out[i] = acc[i];
}

constexpr int kFinCols = 16;       // columns per CTA
constexpr int kFinThreads = 256;
constexpr int kFinSlab = 128;      // chunk partials staged per pass (16 KB)
constexpr int kFinPer = kFinSlab * kFinCols / kFinThreads;

// Stages the partials of 16 columns, kFinSlab chunks at a time, every
// thread's loads in flight together; then thread (column, side) of the
// first warp adds its side's chunks (X or W) in chunk order.
__global__ void __launch_bounds__(kFinThreads) sens_finalize_kernel(SensArgs a, double *H, double *E, double *s) {
  pdl_wait();
  pdl_trigger();
  __shared__ double sp[kFinSlab][kFinCols];
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kFinCols;
  const int nch = a.nchunk_x + a.nchunk_w;
  const int col = threadIdx.x & (kFinCols - 1), side = (threadIdx.x >> 4) & 1;
  double acc = 0.0;
  for (int s0 = 0; s0 < nch; s0 += kFinSlab) {
    const int ns = min(kFinSlab, nch - s0);
    double v[kFinPer];
#pragma unroll
    for (int u = 0; u < kFinPer; ++u) {
      const int i = threadIdx.x + u * kFinThreads, ch = i / kFinCols, cc = i % kFinCols;
      const int64_t c = c0 + cc;
      v[u] = ch < ns && c < a.K ? a.part[static_cast<int64_t>(s0 + ch) * a.K + c] : 0.0;
    }
    __syncthreads();                                   // the previous slab has been summed
#pragma unroll
    for (int u = 0; u < kFinPer; ++u) {
      const int i = threadIdx.x + u * kFinThreads;
      sp[i / kFinCols][i % kFinCols] = v[u];
    }
    __syncthreads();
    if (threadIdx.x < 2 * kFinCols) {
      const int lo = side ? a.nchunk_x : 0, hi = side ? nch : a.nchunk_x;
      const int b0 = max(lo, s0) - s0, b1 = min(hi, s0 + ns) - s0;
      for (int ch = b0; ch < b1; ++ch) acc = __dadd_rn(acc, sp[ch][col]);
    }
  }
  if (threadIdx.x >= 2 * kFinCols) return;
  const double se = __shfl_down_sync(0xffffffffu, acc, kFinCols);
  const int64_t j = c0 + col;
  if (side || j >= a.K) return;
  const double h = __ddiv_rn(__dmul_rn(2.0, acc), static_cast<double>(a.T));
  H[j] = h;
  if (E) E[j] = se;
  s[j] = __dmul_rn(h, se);
}

template <bool XF, bool WF>
static void launch_partials(const SensArgs &a, bool xvec, bool wvec, dim3 grid, cudaStream_t st) {
  if (xvec && wvec) launch_pdl(sens_partial_kernel<XF, WF, true, true>, dim3(grid), dim3(kSensThreads), 0, st, a);
  else if (xvec) launch_pdl(sens_partial_kernel<XF, WF, true, false>, dim3(grid), dim3(kSensThreads), 0, st, a);
  else if (wvec) launch_pdl(sens_partial_kernel<XF, WF, false, true>, dim3(grid), dim3(kSensThreads), 0, st, a);
  else launch_pdl(sens_partial_kernel<XF, WF, false, false>, dim3(grid), dim3(kSensThreads), 0, st, a);
}

static int64_t chunks(int64_t rows) { return (rows + kSumChunk - 1) / kSumChunk; }

}  // namespace mxs

using namespace mxs;

extern "C" mxs_status mxs_sensitivity_workspace_bytes(int64_t T, int64_t N, int64_t K, size_t *bytes) {
  if (!bytes || T < 1 || N < 1 || K < 1) return MXS_ERR_ARG;
  *bytes = static_cast<size_t>((chunks(T) + chunks(N)) * K * 8);
  return MXS_OK;
}

extern "C" mxs_status mxs_sensitivity(const void *X, mxs_dtype xt, int64_t T, int64_t K, int64_t ldx,
                                      const void *W, mxs_dtype wt, int64_t N, int64_t ldw,
                                      double *H, double *E, double *s,
                                      void *ws, size_t ws_bytes, void *stream) {
  if (!X || !W || !H || !s || T < 1 || N < 1 || K < 1) return MXS_ERR_ARG;
  if (!dtype_ok(xt) || !dtype_ok(wt)) return MXS_ERR_DTYPE;
  if (ldx < K || ldw < K) return MXS_ERR_SHAPE;
  if (chunks(T) + chunks(N) > 65535) return MXS_ERR_SHAPE;
  size_t need = 0;
  mxs_sensitivity_workspace_bytes(T, N, K, &need);
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MXS_ERR_WORKSPACE;
  mxs_status st = check_device();
  if (st != MXS_OK) return st;
  SensArgs a{};
  a.X = X;
  a.W = W;
  a.T = T;
  a.N = N;
  a.K = K;
  a.ldx = ldx;
  a.ldw = ldw;
  a.nchunk_x = static_cast<int32_t>(chunks(T));
  a.nchunk_w = static_cast<int32_t>(chunks(N));
  a.part = reinterpret_cast<double *>(ws);
  // vector loads and TMA tiles (4 columns: 8 bytes bf16, 16 bytes fp32) need aligned rows
  const bool xvec = aligned16(X) && (ldx * static_cast<int64_t>(dtype_size(xt))) % 16 == 0;
  const bool wvec = aligned16(W) && (ldw * static_cast<int64_t>(dtype_size(wt))) % 16 == 0;
  const int64_t col_threads = (K + kColsPerThread - 1) / kColsPerThread;
  dim3 grid(static_cast<unsigned>((col_threads + kSensThreads - 1) / kSensThreads),
            static_cast<unsigned>(a.nchunk_x + a.nchunk_w));
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const bool xf = xt == MXS_F32, wf = wt == MXS_F32;
  bool tiled = false;
  if (xvec && wvec) {
    // TMA tiles: 64-row chunks x 256 columns per CTA, in 8-row sub-tiles
    CUtensorMap mx{}, mw{};
    int *status = device_status_word();
    const int64_t ctiles = (K + kTileCols - 1) / kTileCols;
    const int64_t ntiles = (a.nchunk_x + a.nchunk_w) * ctiles;
    if (status && ntiles < (1ll << 31) &&
        make_plain_map(&mx, xf ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                       static_cast<int>(dtype_size(xt)), X, K, T, ldx, kTileCols, kSubRows) &&
        make_plain_map(&mw, wf ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                       static_cast<int>(dtype_size(wt)), W, K, N, ldw, kTileCols, kSubRows)) {
      const int smem = kSubBufs * kSubRows * kTileCols * ((xf || wf) ? 4 : 2);
      const unsigned g = static_cast<unsigned>(ntiles);
      const int32_t ct = static_cast<int32_t>(ctiles);
      if (xf && wf) {
        if (!ensure_smem(sens_tile_kernel<true, true>, smem)) return MXS_ERR_CUDA;
        launch_pdl(sens_tile_kernel<true, true>, dim3(g), dim3(kTileThreads), smem, cs, mx, mw, a, ct, status);
      } else if (xf) {
        if (!ensure_smem(sens_tile_kernel<true, false>, smem)) return MXS_ERR_CUDA;
        launch_pdl(sens_tile_kernel<true, false>, dim3(g), dim3(kTileThreads), smem, cs, mx, mw, a, ct, status);
      } else if (wf) {
        if (!ensure_smem(sens_tile_kernel<false, true>, smem)) return MXS_ERR_CUDA;
        launch_pdl(sens_tile_kernel<false, true>, dim3(g), dim3(kTileThreads), smem, cs, mx, mw, a, ct, status);
      } else {
        launch_pdl(sens_tile_kernel<false, false>, dim3(g), dim3(kTileThreads), smem, cs, mx, mw, a, ct, status);
      }
      tiled = true;
    }
  }
  if (!tiled) {
    if (xf && wf) launch_partials<true, true>(a, xvec, wvec, grid, cs);
    else if (xf) launch_partials<true, false>(a, xvec, wvec, grid, cs);
    else if (wf) launch_partials<false, true>(a, xvec, wvec, grid, cs);
    else launch_partials<false, false>(a, xvec, wvec, grid, cs);
  }
  launch_pdl(sens_finalize_kernel, dim3(static_cast<unsigned>((K + kFinCols - 1) / kFinCols)), dim3(kFinThreads), 0, cs, a, H, E, s);
  count_launch(2);
  return cuda_status(cudaGetLastError());
}

// ------------------------------------------------------- no-allocation entry
//
// Some callers cannot call cudaMalloc at all: code running inside CUDA stream
// capture (allocation is not a capturable stream operation), runtimes that
// hand a library no allocator, and latency-critical paths that must not take
// the allocator's locks.  For them the chunk partials live in one file-scope
// device array of fixed size instead of a caller-provided workspace.
namespace mxs {

constexpr size_t kNoAllocScratchBytes = MXS_NOALLOC_SCRATCH_BYTES;   // 16 MiB: 2 Mi chunk partials
__device__ __align__(256) uint8_t g_sens_scratch[kNoAllocScratchBytes];

// Address of the scratch array in the current device's context.  It is
// looked up once per device with that device current, and again only when
// the context has changed since (a device reset destroys the context, and
// the module's arrays move with the new one).
static mxs_status sens_scratch(void **ptr) {
  struct Entry {
    unsigned long long ctx;
    void *addr;
  };
  static Entry cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MXS_ERR_CUDA;
  if (dev < 0 || dev >= 64) return MXS_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (!ctx || cache[dev].ctx != ctx || !cache[dev].addr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sens_scratch) != cudaSuccess || !p) return MXS_ERR_CUDA;
    cache[dev] = Entry{current_context_id(), p};
  }
  *ptr = cache[dev].addr;
  return MXS_OK;
}

}  // namespace mxs

extern "C" mxs_status mxs_sensitivity_noalloc(const void *X, mxs_dtype xt, int64_t T, int64_t K, int64_t ldx,
                                              const void *W, mxs_dtype wt, int64_t N, int64_t ldw,
                                              double *H, double *E, double *s, void *stream) {
  // the same argument checks as mxs_sensitivity, in the same order, before
  // anything touches the device
  if (!X || !W || !H || !s || T < 1 || N < 1 || K < 1) return MXS_ERR_ARG;
  if (!dtype_ok(xt) || !dtype_ok(wt)) return MXS_ERR_DTYPE;
  if (ldx < K || ldw < K) return MXS_ERR_SHAPE;
  if (chunks(T) + chunks(N) > 65535) return MXS_ERR_SHAPE;
  size_t need = 0;
  mxs_status st = mxs_sensitivity_workspace_bytes(T, N, K, &need);
  if (st != MXS_OK) return st;
  if (need > kNoAllocScratchBytes) return MXS_ERR_WORKSPACE;   // shape needs more than the fixed scratch
  void *scratch = nullptr;
  if ((st = check_device()) != MXS_OK) return st;
  if ((st = sens_scratch(&scratch)) != MXS_OK) return st;
  // every partial the finalize pass reads is written earlier in the same
  // call, so nothing in the scratch has to start at zero
  return mxs_sensitivity(X, xt, T, K, ldx, W, wt, N, ldw, H, E, s, scratch, kNoAllocScratchBytes, stream);
}
