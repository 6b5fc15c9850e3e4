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
// fp64; chunk sums are then added in chunk order.  Each term is one fp64
// product (a square of an fp32/bf16 value, exact; or of the exact fp64
// difference W - Q4(W)), formed and added with explicit round-to-nearest
// intrinsics so that no fused multiply-add can change the result.
//
// Two launches: (1) partial sums, one CTA row per 64-row chunk of X or of W,
// each thread owning 8 consecutive columns (16-byte bf16 / 32-byte fp32
// loads, coalesced across the warp); for W the 4 lanes that own one 32-column
// block share its maximum through two xor-shuffles; (2) a per-column pass that
// adds the chunk sums in order and forms H, E and s.
#include <algorithm>

#include "mxs_internal.cuh"

namespace mxs {

constexpr int kSumChunk = 64;
constexpr int kSensThreads = 256;
constexpr int kColsPerThread = 8;

struct SensArgs {
  const void *X;
  const void *W;
  int64_t T, N, K, ldx, ldw;
  int32_t nchunk_x, nchunk_w;
  double *part;        // (nchunk_x + nchunk_w) x K
};

template <bool F32, bool VEC>
__device__ __forceinline__ void load8(const void *base, int64_t row_off, int64_t c0, int64_t K,
                                      float (&v)[kColsPerThread]) {
  if (VEC && c0 + kColsPerThread <= K) {
    if constexpr (F32) {
      const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + row_off + c0);
      float4 a = __ldg(p), b = __ldg(p + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
      uint4 a = __ldg(reinterpret_cast<const uint4 *>(reinterpret_cast<const unsigned short *>(base) + row_off + c0));
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
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

template <bool XF32, bool WF32, bool XVEC, bool WVEC>
__global__ void __launch_bounds__(kSensThreads) sens_partial_kernel(SensArgs a) {
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
    for (int64_t t = r0; t < r1; ++t) {
      float v[kColsPerThread];
      load8<XF32, XVEC>(a.X, t * a.ldx, c0, a.K, v);
#pragma unroll
      for (int i = 0; i < kColsPerThread; ++i) {
        const double x = static_cast<double>(v[i]);
        acc[i] = __dadd_rn(acc[i], __dmul_rn(x, x));
      }
    }
  } else {
    // All lanes stay to the end: the block maximum needs the 4 owner lanes.
    const int wchunk = chunk - a.nchunk_x;
    const int64_t r0 = static_cast<int64_t>(wchunk) * kSumChunk;
    const int64_t r1 = min(r0 + kSumChunk, a.N);
    for (int64_t i = r0; i < r1; ++i) {
      float v[kColsPerThread];
      load8<WF32, WVEC>(a.W, i * a.ldw, c0, a.K, v);
      uint32_t amax = 0;
#pragma unroll
      for (int t = 0; t < kColsPerThread; ++t) amax = max(amax, __float_as_uint(v[t]) & 0x7fffffffu);
      amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const int ef = static_cast<int>(amax >> 23);
      const int e = ef == 0 ? -127 : ef - 127;
      const double step = pow2d(e - 2);
#pragma unroll
      for (int t = 0; t < kColsPerThread; ++t) {
        int q = __float2int_rn(scale_pow2(v[t], 2 - e));
        q = min(max(q, -7), 7);
        const double d = __dsub_rn(static_cast<double>(v[t]), __dmul_rn(static_cast<double>(q), step));
        acc[t] = __dadd_rn(acc[t], __dmul_rn(d, d));
      }
    }
    if (c0 >= a.K) return;
  }
  double *out = a.part + static_cast<int64_t>(chunk) * a.K + c0;
#pragma unroll
  for (int i = 0; i < kColsPerThread; ++i)
    if (c0 + i < a.K) out[i] = acc[i];
}

__global__ void sens_finalize_kernel(SensArgs a, double *H, double *E, double *s) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= a.K) return;
  double sx = 0.0;
  for (int c = 0; c < a.nchunk_x; ++c) sx = __dadd_rn(sx, a.part[static_cast<int64_t>(c) * a.K + j]);
  double se = 0.0;
  for (int c = 0; c < a.nchunk_w; ++c)
    se = __dadd_rn(se, a.part[static_cast<int64_t>(a.nchunk_x + c) * a.K + j]);
  const double h = __ddiv_rn(__dmul_rn(2.0, sx), static_cast<double>(a.T));
  H[j] = h;
  if (E) E[j] = se;
  s[j] = __dmul_rn(h, se);
}

template <bool XF, bool WF>
static void launch_partials(const SensArgs &a, bool xvec, bool wvec, dim3 grid, cudaStream_t st) {
  if (xvec && wvec) sens_partial_kernel<XF, WF, true, true><<<grid, kSensThreads, 0, st>>>(a);
  else if (xvec) sens_partial_kernel<XF, WF, true, false><<<grid, kSensThreads, 0, st>>>(a);
  else if (wvec) sens_partial_kernel<XF, WF, false, true><<<grid, kSensThreads, 0, st>>>(a);
  else sens_partial_kernel<XF, WF, false, false><<<grid, kSensThreads, 0, st>>>(a);
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
  // 16-byte vector loads need aligned rows: base and pitch multiples of 16 bytes.
  const bool xvec = aligned16(X) && (ldx * static_cast<int64_t>(dtype_size(xt))) % 16 == 0;
  const bool wvec = aligned16(W) && (ldw * static_cast<int64_t>(dtype_size(wt))) % 16 == 0;
  const int64_t col_threads = (K + kColsPerThread - 1) / kColsPerThread;
  dim3 grid(static_cast<unsigned>((col_threads + kSensThreads - 1) / kSensThreads),
            static_cast<unsigned>(a.nchunk_x + a.nchunk_w));
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const bool xf = xt == MXS_F32, wf = wt == MXS_F32;
  if (xf && wf) launch_partials<true, true>(a, xvec, wvec, grid, cs);
  else if (xf) launch_partials<true, false>(a, xvec, wvec, grid, cs);
  else if (wf) launch_partials<false, true>(a, xvec, wvec, grid, cs);
  else launch_partials<false, false>(a, xvec, wvec, grid, cs);
  sens_finalize_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, cs>>>(a, H, E, s);
  count_launch(2);
  return cuda_status(cudaGetLastError());
}
