// mxs_stack.cu -- layer-wise sensitivity scores of a decoder stack.
//
// MXSens (arXiv 2607.17733), technical summary §2.1 "Laaggewijze
// Sensitiviteit": a layer's score is the L2 error at the model's final
// output when that layer alone is quantised; §2.3 "Dynamische 6-bit
// Allocatie" turns the scores into 6-bit counts (mxs_allocate's
// MXS_ALLOC_LAYER mode).
//
// The model is the Llama decoder stack of the workload, random-initialised:
// synthetic hidden states in, final-normed hidden states out (no embedding
// table or LM head).  Block: RMSNorm (weight 1) -> q, k, v projections ->
// rotary embedding (rotate-half form) -> causal grouped-query softmax
// attention -> o projection + residual -> RMSNorm -> silu(gate) * up -> down
// projection + residual; a final RMSNorm gives the output.  Everything runs
// in fp32 on the GPU, except the one linear being scored, which runs as the
// library's W4A4 MXINT4 layer: mxs_quantize_act of its fp32 input and
// mxs_quantize_weight of its bf16 weight in the uniform 4-bit layout, then
// mxs_gemm (bf16 output).
//
// Schedule: one unquantised pass stores every block's input; the score of
// linear j of block b restarts from block b's stored input, runs block b with
// linear j quantised and the later blocks unquantised, and reduces
// ||F_q - F||^2 in fp64 (fixed order, so the score does not depend on the
// launch).  The fp32 linears use a register-tiled SIMT kernel that reads the
// bf16 weights directly (exact bf16 -> fp32 widening, fp32 products and
// sums), so the reference forward is an fp32 computation of the stack.
#include <algorithm>
#include <cmath>
#include <vector>

#include "mxs_internal.cuh"

namespace mxs {
namespace {

constexpr int kLinears = 7;                 // q, k, v, o, gate, up, down
constexpr int kMaxTokens = 1024;
constexpr int kGemmBT = 64, kGemmBN = 64, kGemmBK = 32, kGemmThreads = 256;
constexpr int kScoreParts = 296;

struct Dims {
  int64_t T, hidden, n_heads, n_kv, hd, mlp;
  // (N, K) of linear j
  int64_t N(int j) const {
    return j == 0 ? n_heads * hd : (j <= 2 ? n_kv * hd : (j == 3 || j == 6 ? hidden : mlp));
  }
  int64_t K(int j) const { return j == 3 ? n_heads * hd : (j == 6 ? mlp : hidden); }
};

// ------------------------------------------------------------------ kernels

// y = x / sqrt(mean(x^2) + eps) per row; the mean square is summed in fp64.
__global__ void __launch_bounds__(256) rms_kernel(const float *x, float *y, int64_t D, float eps) {
  pdl_wait();
  pdl_trigger();
  __shared__ double red[8];
  const float *xr = x + blockIdx.x * D;
  float *yr = y + blockIdx.x * D;
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < D; i += 256) s += static_cast<double>(xr[i]) * xr[i];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < 8; ++w) t += red[w];
  const float r = static_cast<float>(1.0 / sqrt(t / static_cast<double>(D) + static_cast<double>(eps)));
  for (int64_t i = threadIdx.x; i < D; i += 256) yr[i] = xr[i] * r;
}

// Y[t][n] (+)= sum_k X[t][k] * W[n][k]; X fp32 (pitch ldx), W bf16 (K per
// row), Y fp32 (pitch ldy).  64 x 64 output tile per CTA, 4 x 4 per thread,
// K in steps of 32 staged (transposed) in shared memory.  K % 32 == 0.
__global__ void __launch_bounds__(kGemmThreads) gemm_f32_kernel(const float *X, int64_t ldx,
                                                                const __nv_bfloat16 *W, float *Y, int64_t ldy,
                                                                int64_t T, int64_t N, int64_t K, int accumulate) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) float xs[kGemmBK][kGemmBT + 4];
  __shared__ __align__(16) float ws[kGemmBK][kGemmBN + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kGemmBT, n0 = static_cast<int64_t>(blockIdx.x) * kGemmBN;
  float acc[4][4] = {};
  // loader: row r = tid / 4 (0..63), 8 consecutive k at c = 8 (tid % 4)
  const int lr = tid >> 2, lc = 8 * (tid & 3);
  for (int64_t k0 = 0; k0 < K; k0 += kGemmBK) {
    float xv[8], wv[8];
    if (t0 + lr < T) {
      const float4 *p = reinterpret_cast<const float4 *>(X + (t0 + lr) * ldx + k0 + lc);
      const float4 a = p[0], b = p[1];
      xv[0] = a.x; xv[1] = a.y; xv[2] = a.z; xv[3] = a.w; xv[4] = b.x; xv[5] = b.y; xv[6] = b.z; xv[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) xv[i] = 0.f;
    }
    if (n0 + lr < N) {
      const uint4 q = *reinterpret_cast<const uint4 *>(W + (n0 + lr) * K + k0 + lc);
      const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        wv[2 * i] = __uint_as_float(w4[i] << 16);
        wv[2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) wv[i] = 0.f;
    }
    __syncthreads();                                   // the previous tile has been read
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      xs[lc + i][lr] = xv[i];
      ws[lc + i][lr] = wv[i];
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kGemmBK; ++k) {
      const float4 a = *reinterpret_cast<const float4 *>(&xs[k][4 * ty]);
      const float4 b = *reinterpret_cast<const float4 *>(&ws[k][4 * tx]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = t0 + 4 * ty + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + 4 * tx + j;
      if (n < N) Y[t * ldy + n] = accumulate ? Y[t * ldy + n] + acc[i][j] : acc[i][j];
    }
  }
}

// Rotary embedding in place on a T x (heads * d) projection: token t, head
// h, pair (i, i + d/2) turns by t * theta^(-2i/d) (angle and its sine and
// cosine in fp64).
__global__ void rope_kernel(float *x, int64_t T, int heads, int d, double theta) {
  pdl_wait();
  pdl_trigger();
  const int half = d / 2;
  const int64_t total = T * heads * half;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(idx % half);
    const int64_t th = idx / half;
    const int h = static_cast<int>(th % heads);
    const int64_t t = th / heads;
    const double ang = static_cast<double>(t) * pow(theta, -2.0 * i / d);
    double s, c;
    sincos(ang, &s, &c);
    float *p = x + t * static_cast<int64_t>(heads) * d + static_cast<int64_t>(h) * d;
    const float a = p[i], b = p[i + half];
    p[i] = static_cast<float>(a * c - b * s);
    p[i + half] = static_cast<float>(a * s + b * c);
  }
}

// Causal grouped-query attention, one CTA per (token t, query head h), four
// warps: warp w scores keys w, w + 4, ... (dot products across the lanes),
// then softmax over keys 0..t and the weighted sum of the value rows.
__global__ void __launch_bounds__(128) attn_prefill_kernel(const float *q, const float *k, const float *v, float *o,
                                                           int64_t T, int heads, int kv_heads, int d, float scale) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s[kMaxTokens];
  __shared__ float qs[256];
  __shared__ float red[4];
  const int t = blockIdx.x, h = blockIdx.y, g = h / (heads / kv_heads);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t qw = static_cast<int64_t>(heads) * d, kw = static_cast<int64_t>(kv_heads) * d;
  for (int i = threadIdx.x; i < d; i += 128) qs[i] = q[t * qw + static_cast<int64_t>(h) * d + i];
  __syncthreads();
  for (int u = warp; u <= t; u += 4) {
    const float *kr = k + u * kw + static_cast<int64_t>(g) * d;
    float dot = 0.f;
    for (int i = lane; i < d; i += 32) dot = fmaf(qs[i], kr[i], dot);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    if (lane == 0) s[u] = dot * scale;
  }
  __syncthreads();
  float m = -INFINITY;
  for (int u = threadIdx.x; u <= t; u += 128) m = fmaxf(m, s[u]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float sum = 0.f;
  for (int u = threadIdx.x; u <= t; u += 128) {
    const float p = expf(s[u] - m);
    s[u] = p;
    sum += p;
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane == 0) red[warp] = sum;
  __syncthreads();
  sum = (red[0] + red[1]) + (red[2] + red[3]);
  for (int i = threadIdx.x; i < d; i += 128) {
    const float *vr = v + static_cast<int64_t>(g) * d + i;
    float acc = 0.f;
    for (int u = 0; u <= t; ++u) acc = fmaf(s[u], vr[u * kw], acc);
    o[t * qw + static_cast<int64_t>(h) * d + i] = acc / sum;
  }
}

// m = silu(g) * u = g / (1 + e^-g) * u.
__global__ void swiglu_kernel(const float *g, const float *u, float *m, int64_t n) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float x = g[i];
    m[i] = x / (1.f + expf(-x)) * u[i];
  }
}

// out (+)= float(y) for a T x N bf16 matrix (pitch N) into pitch ldo.
__global__ void widen_kernel(const __nv_bfloat16 *y, float *out, int64_t ldo, int64_t T, int64_t N, int accumulate) {
  pdl_wait();
  pdl_trigger();
  const int64_t total = T * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / N, n = i - t * N;
    const float v = __bfloat162float(y[i]);
    out[t * ldo + n] = accumulate ? out[t * ldo + n] + v : v;
  }
}

// partial[b] = sum over a fixed stride of (a - b)^2 in fp64; the finishing
// kernel adds the partials in order and writes the root.
__global__ void __launch_bounds__(256) sqdiff_kernel(const float *a, const float *b, int64_t n, double *partial) {
  pdl_wait();
  pdl_trigger();
  __shared__ double red[8];
  double s = 0.0;
  for (int64_t i = blockIdx.x * 256 + threadIdx.x; i < n; i += static_cast<int64_t>(gridDim.x) * 256) {
    const double d = static_cast<double>(a[i]) - static_cast<double>(b[i]);
    s = fma(d, d, s);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += red[w];
    partial[blockIdx.x] = t;
  }
}

__global__ void score_finish_kernel(const double *partial, int nparts, double *score) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < nparts; ++i) t += partial[i];
    *score = sqrt(t);
  }
}

// ------------------------------------------------------------------- host

struct Ws {
  float *hin, *h, *a, *q, *k, *v, *att, *g, *u, *fref, *fq;
  __nv_bfloat16 *ybf;
  uint8_t *aq_codes, *aq_scales, *wq_codes, *wq_scales, *gemm_ws;
  double *partial, *scores;
  size_t gemm_ws_bytes, total;
};

int64_t pitch16(int64_t b) { return round_up(b, 16); }

// Uniform 4-bit tensor over caller buffers (rows x K).
mxs_mxtensor uniform4(int64_t rows, int64_t K, uint8_t *codes, uint8_t *scales) {
  mxs_mxtensor t{};
  const int64_t counts[3] = {0, 0, K};
  mxs_layout_make(K, counts, nullptr, &t.lay);
  t.rows = rows;
  t.codes[2] = codes;
  t.scales[2] = scales;
  t.code_pitch[2] = pitch16(pad32(K) / 2);
  t.scale_pitch[2] = pitch16(pad32(K) / 32);
  return t;
}

Ws plan(const Dims &D, int64_t n_blocks, uint8_t *base) {
  Ws w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t *p = base ? base + off : nullptr;
    off += static_cast<size_t>(round_up(static_cast<int64_t>(bytes), 256));
    return p;
  };
  const int64_t T = D.T, wide = std::max(D.hidden, std::max(D.mlp, D.n_heads * D.hd));
  int64_t nk_max = 0, n_max = 0, k_max = 0, gws = 0;
  for (int j = 0; j < kLinears; ++j) {
    nk_max = std::max(nk_max, D.N(j) * pitch16(pad32(D.K(j)) / 2) + D.N(j) * pitch16(pad32(D.K(j)) / 32));
    n_max = std::max(n_max, D.N(j));
    k_max = std::max(k_max, D.K(j));
    // the GEMM's workspace for this shape (host-side size query only)
    uint8_t *fake = reinterpret_cast<uint8_t *>(uintptr_t(1) << 20);
    mxs_mxtensor A = uniform4(T, D.K(j), fake, fake), Wt = uniform4(D.N(j), D.K(j), fake, fake);
    size_t b = 0;
    if (mxs_gemm_workspace_bytes(&A, &Wt, &b) == MXS_OK) gws = std::max<int64_t>(gws, static_cast<int64_t>(b));
  }
  w.hin = reinterpret_cast<float *>(take(static_cast<size_t>(n_blocks * T * D.hidden * 4)));
  w.h = reinterpret_cast<float *>(take(static_cast<size_t>(T * D.hidden * 4)));
  w.a = reinterpret_cast<float *>(take(static_cast<size_t>(T * wide * 4)));
  w.q = reinterpret_cast<float *>(take(static_cast<size_t>(T * D.n_heads * D.hd * 4)));
  w.k = reinterpret_cast<float *>(take(static_cast<size_t>(T * D.n_kv * D.hd * 4)));
  w.v = reinterpret_cast<float *>(take(static_cast<size_t>(T * D.n_kv * D.hd * 4)));
  w.att = reinterpret_cast<float *>(take(static_cast<size_t>(T * D.n_heads * D.hd * 4)));
  w.g = reinterpret_cast<float *>(take(static_cast<size_t>(T * D.mlp * 4)));
  w.u = reinterpret_cast<float *>(take(static_cast<size_t>(T * D.mlp * 4)));
  w.fref = reinterpret_cast<float *>(take(static_cast<size_t>(T * D.hidden * 4)));
  w.fq = reinterpret_cast<float *>(take(static_cast<size_t>(T * D.hidden * 4)));
  w.ybf = reinterpret_cast<__nv_bfloat16 *>(take(static_cast<size_t>(T * n_max * 2)));
  w.aq_codes = take(static_cast<size_t>(T * pitch16(pad32(k_max) / 2)));
  w.aq_scales = take(static_cast<size_t>(T * pitch16(pad32(k_max) / 32)));
  w.wq_codes = take(static_cast<size_t>(nk_max));
  w.wq_scales = nullptr;                               // placed after the codes of each matrix
  w.gemm_ws_bytes = static_cast<size_t>(gws);
  w.gemm_ws = take(static_cast<size_t>(std::max<int64_t>(gws, 256)) + 1024);
  if (w.gemm_ws)                                       // mxs_gemm wants a 1024-byte aligned workspace
    w.gemm_ws = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(w.gemm_ws) + 1023) & ~uintptr_t(1023));
  w.partial = reinterpret_cast<double *>(take(kScoreParts * 8));
  w.scores = reinterpret_cast<double *>(take(static_cast<size_t>(n_blocks * kLinears * 8)));
  w.total = off;
  return w;
}

struct Runner {
  const mxs_stack *m;
  Dims D;
  Ws w;
  cudaStream_t cs;
  mxs_status st = MXS_OK;

  void fail(mxs_status s) {
    if (st == MXS_OK) st = s;
  }
  void launched(int n = 1) {
    count_launch(n);
    if (cudaGetLastError() != cudaSuccess) fail(MXS_ERR_CUDA);
  }
  const __nv_bfloat16 *weight(int64_t b, int j) const {
    return static_cast<const __nv_bfloat16 *>(m->W[kLinears * b + j]);
  }
  void rms(const float *x, float *y) {
    launch_pdl(rms_kernel, dim3(static_cast<unsigned>(D.T)), dim3(256), 0, cs, x, y, D.hidden, m->rms_eps);
    launched();
  }
  // out (+)= x W^T for linear j of block b, fp32 or (quant) the W4A4 layer
  void linear(int64_t b, int j, const float *x, float *out, int64_t ldo, bool accumulate, bool quant) {
    const int64_t N = D.N(j), K = D.K(j);
    if (!quant) {
      dim3 grid(static_cast<unsigned>((N + kGemmBN - 1) / kGemmBN), static_cast<unsigned>((D.T + kGemmBT - 1) / kGemmBT));
      launch_pdl(gemm_f32_kernel, grid, dim3(kGemmThreads), 0, cs, x, K, weight(b, j), out, ldo, D.T, N, K,
                 accumulate ? 1 : 0);
      launched();
      return;
    }
    mxs_mxtensor Wq = uniform4(N, K, w.wq_codes, nullptr);
    Wq.scales[2] = w.wq_codes + N * Wq.code_pitch[2];
    mxs_mxtensor Aq = uniform4(D.T, K, w.aq_codes, w.aq_scales);
    mxs_status s;
    if ((s = mxs_quantize_weight(weight(b, j), MXS_BF16, N, K, &Wq, cs)) != MXS_OK) return fail(s);
    if ((s = mxs_quantize_act(x, MXS_F32, D.T, K, &Aq, cs)) != MXS_OK) return fail(s);
    if ((s = mxs_gemm(&Aq, &Wq, w.ybf, N, w.gemm_ws, w.gemm_ws_bytes, cs)) != MXS_OK) return fail(s);
    const int64_t total = D.T * N;
    launch_pdl(widen_kernel, dim3(static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, 4096))), dim3(256), 0,
               cs, static_cast<const __nv_bfloat16 *>(w.ybf), out, ldo, D.T, N, accumulate ? 1 : 0);
    launched();
  }
  void block(int64_t b, int quant) {
    const int64_t T = D.T, qw = D.n_heads * D.hd, kw = D.n_kv * D.hd;
    rms(w.h, w.a);
    linear(b, 0, w.a, w.q, qw, false, quant == 0);
    linear(b, 1, w.a, w.k, kw, false, quant == 1);
    linear(b, 2, w.a, w.v, kw, false, quant == 2);
    const int rgrid = static_cast<int>(std::min<int64_t>((T * D.n_heads * D.hd / 2 + 255) / 256, 4096));
    launch_pdl(rope_kernel, dim3(rgrid), dim3(256), 0, cs, w.q, T, static_cast<int>(D.n_heads),
               static_cast<int>(D.hd), static_cast<double>(m->rope_theta));
    launch_pdl(rope_kernel, dim3(rgrid), dim3(256), 0, cs, w.k, T, static_cast<int>(D.n_kv), static_cast<int>(D.hd),
               static_cast<double>(m->rope_theta));
    launched(2);
    launch_pdl(attn_prefill_kernel, dim3(static_cast<unsigned>(T), static_cast<unsigned>(D.n_heads)), dim3(128), 0, cs,
               static_cast<const float *>(w.q), static_cast<const float *>(w.k), static_cast<const float *>(w.v),
               w.att, T, static_cast<int>(D.n_heads), static_cast<int>(D.n_kv), static_cast<int>(D.hd),
               static_cast<float>(1.0 / std::sqrt(static_cast<double>(D.hd))));
    launched();
    linear(b, 3, w.att, w.h, D.hidden, true, quant == 3);
    rms(w.h, w.a);
    linear(b, 4, w.a, w.g, D.mlp, false, quant == 4);
    linear(b, 5, w.a, w.u, D.mlp, false, quant == 5);
    const int64_t n = T * D.mlp;
    launch_pdl(swiglu_kernel, dim3(static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 4096))), dim3(256), 0, cs,
               static_cast<const float *>(w.g), static_cast<const float *>(w.u), w.a, n);
    launched();
    linear(b, 6, w.a, w.h, D.hidden, true, quant == 6);
  }
  void score(int64_t l) {
    rms(w.h, w.fq);
    launch_pdl(sqdiff_kernel, dim3(kScoreParts), dim3(256), 0, cs, static_cast<const float *>(w.fq),
               static_cast<const float *>(w.fref), D.T * D.hidden, w.partial);
    launch_pdl(score_finish_kernel, dim3(1), dim3(32), 0, cs, static_cast<const double *>(w.partial), kScoreParts,
               w.scores + l);
    launched(2);
  }
};

bool dims_of(const mxs_stack *m, int64_t T, Dims *D) {
  if (!m || !m->W || m->n_blocks < 1 || m->hidden < 1 || m->n_heads < 1 || m->n_kv_heads < 1 || m->mlp < 1)
    return false;
  D->T = T;
  D->hidden = m->hidden;
  D->n_heads = m->n_heads;
  D->n_kv = m->n_kv_heads;
  D->hd = m->hidden / m->n_heads;
  D->mlp = m->mlp;
  return true;
}

}  // namespace
}  // namespace mxs

using namespace mxs;

extern "C" mxs_status mxs_layer_scores_workspace_bytes(const mxs_stack *m, int64_t T, size_t *bytes) {
  Dims D{};
  if (!bytes || !dims_of(m, T, &D) || T < 1) return MXS_ERR_ARG;
  if (D.hidden % D.n_heads || D.n_heads % D.n_kv || D.hd % 2 || D.hd > 256 || D.hidden % 32 || D.mlp % 32 ||
      (D.n_heads * D.hd) % 32 || T > kMaxTokens || !std::isfinite(m->rms_eps) || !(m->rope_theta > 0.f))
    return MXS_ERR_SHAPE;
  *bytes = plan(D, m->n_blocks, nullptr).total;
  return MXS_OK;
}

extern "C" mxs_status mxs_layer_scores(const mxs_stack *m, const float *x, int64_t T, int64_t ldx, double *scores,
                                       void *ws, size_t ws_bytes, void *stream) {
  size_t need = 0;
  mxs_status st = mxs_layer_scores_workspace_bytes(m, T, &need);
  if (st != MXS_OK) return st;
  if (!x || !scores) return MXS_ERR_ARG;
  if (ldx < m->hidden) return MXS_ERR_SHAPE;
  for (int64_t i = 0; i < static_cast<int64_t>(m->n_blocks) * kLinears; ++i)
    if (!m->W[i]) return MXS_ERR_ARG;
    else if (!aligned16(m->W[i])) return MXS_ERR_ALIGN;
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MXS_ERR_WORKSPACE;
  if ((st = check_device()) != MXS_OK) return st;
  Runner r{};
  r.m = m;
  dims_of(m, T, &r.D);
  r.w = plan(r.D, m->n_blocks, static_cast<uint8_t *>(ws));
  r.cs = static_cast<cudaStream_t>(stream);
  const int64_t hbytes = T * r.D.hidden * 4;
  // the unquantised pass: every block's input, then the reference output
  if (cudaMemcpy2DAsync(r.w.h, static_cast<size_t>(r.D.hidden * 4), x, static_cast<size_t>(ldx * 4),
                        static_cast<size_t>(r.D.hidden * 4), static_cast<size_t>(T), cudaMemcpyDeviceToDevice,
                        r.cs) != cudaSuccess)
    return MXS_ERR_CUDA;
  for (int64_t b = 0; b < m->n_blocks; ++b) {
    if (cudaMemcpyAsync(r.w.hin + b * T * r.D.hidden, r.w.h, static_cast<size_t>(hbytes), cudaMemcpyDeviceToDevice,
                        r.cs) != cudaSuccess)
      return MXS_ERR_CUDA;
    r.block(b, -1);
  }
  r.rms(r.w.h, r.w.fref);
  // one pass per linear layer, from its block's stored input
  for (int64_t b = 0; b < m->n_blocks && r.st == MXS_OK; ++b) {
    for (int j = 0; j < kLinears && r.st == MXS_OK; ++j) {
      if (cudaMemcpyAsync(r.w.h, r.w.hin + b * T * r.D.hidden, static_cast<size_t>(hbytes), cudaMemcpyDeviceToDevice,
                          r.cs) != cudaSuccess)
        return MXS_ERR_CUDA;
      r.block(b, j);
      for (int64_t b2 = b + 1; b2 < m->n_blocks; ++b2) r.block(b2, -1);
      r.score(kLinears * b + j);
    }
  }
  if (r.st != MXS_OK) return r.st;
  if (cudaMemcpyAsync(scores, r.w.scores, static_cast<size_t>(m->n_blocks * kLinears * 8), cudaMemcpyDeviceToHost,
                      r.cs) != cudaSuccess ||
      cudaStreamSynchronize(r.cs) != cudaSuccess)
    return MXS_ERR_CUDA;
  return MXS_OK;
}
