// mxs_quantize.cu -- mixed-width MXINT quantisers (weights, activations, K/V
// cache) and the decoder, plus the layout helpers of the C ABI.
//
// MXSens (arXiv 2607.17733), technical summary §2.2 (triplet 4/6/8 mantissa
// widths) and §2.3 last paragraph (the widths live inside MXINT's 32-value
// blocks); researchpod summary (widths apply to weights and activations);
// §4 (W4A4KV4: the K/V cache is quantised too).
//
// Coding rule for a block x[0..31] at width m (a fixed reading; the pages
// give the block structure but no formula):
//   e = floor(log2 max|x|) clamped to [-127, 127] (-127 for a zero block),
//       read from the float exponent field: for a normal max the field is
//       e + 127 and it is exactly the E8M0 scale byte; a zero or subnormal
//       max has field 0 = byte for e = -127;
//   q = clamp(rint_half_even(x * 2^(m-2-e)), -(2^(m-1)-1), 2^(m-1)-1),
//       the scaling by a power of two being exact.
//
// Kernel shape: one thread codes one 32-position block (a 32-lane warp covers
// 32 consecutive blocks), so the max is a register reduction and each thread
// emits its packed block with 16/8-byte stores that are contiguous across
// the warp.  With a permutation, a CTA stages the permutation once (padded to
// 33 words per 32 so that the per-thread strided reads are bank-conflict
// free) and each source row once, then gathers from shared memory.
#include <algorithm>
#include <cstdio>
#include <mutex>

#include "mxs_internal.cuh"

namespace mxs {

static int64_t g_launches = 0;
static std::mutex g_launch_mu;

void count_launch(int n) {
  std::lock_guard<std::mutex> lk(g_launch_mu);
  g_launches += n;
}

mxs_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MXS_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MXS_ERR_CUDA;
  return major == 10 ? MXS_OK : MXS_ERR_DEVICE;
}

static int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

mxs_status check_layout(const mxs_layout *lay) {
  if (!lay || lay->K < 0) return MXS_ERR_ARG;
  int64_t off = 0, real = 0;
  for (int g = 0; g < 3; ++g) {
    const mxs_segment &s = lay->seg[g];
    if (s.bits != kSegBits[g] || s.k_real < 0 || s.k_pad != pad32(s.k_real) || s.k_off != off)
      return MXS_ERR_SHAPE;
    off += s.k_pad;
    real += s.k_real;
  }
  if (real != lay->K || off != lay->K_pad) return MXS_ERR_SHAPE;
  return MXS_OK;
}

mxs_status check_mxtensor(const mxs_mxtensor *t) {
  if (!t || t->rows < 0) return MXS_ERR_ARG;
  mxs_status st = check_layout(&t->lay);
  if (st != MXS_OK) return st;
  for (int g = 0; g < 3; ++g) {
    const mxs_segment &s = t->lay.seg[g];
    if (s.k_pad == 0 || t->rows == 0) continue;
    if (!t->codes[g] || !t->scales[g]) return MXS_ERR_ARG;
    if (!aligned16(t->codes[g]) || !aligned16(t->scales[g])) return MXS_ERR_ALIGN;
    if (t->code_pitch[g] % 16 || t->scale_pitch[g] % 16) return MXS_ERR_ALIGN;
    if (t->code_pitch[g] < seg_row_bytes(s.k_pad, s.bits) || t->scale_pitch[g] < s.k_pad / kBlock)
      return MXS_ERR_SHAPE;
  }
  return MXS_OK;
}

// ------------------------------------------------------------------ kernels

struct QuantArgs {
  const void *src;
  int64_t ld;          // elements
  int64_t rows, K;
  const int32_t *perm; // NULL: identity
  int64_t k_real[3];
  int64_t real_off[3]; // first real position of each segment in perm order
  int32_t nb[3];       // blocks per row per segment
  int32_t nb_total;
  uint8_t *codes[3];
  int64_t cpitch[3];
  uint8_t *scales[3];
  int64_t spitch[3];
};

template <int M>
__device__ __forceinline__ void encode_store(const float (&v)[kBlock], uint8_t *cdst, uint8_t *sdst) {
  uint32_t amax = 0;
#pragma unroll
  for (int t = 0; t < kBlock; ++t) amax = max(amax, __float_as_uint(v[t]) & 0x7fffffffu);
  const int ef = static_cast<int>(amax >> 23);   // E8M0 byte of the block
  const int e = ef == 0 ? -127 : ef - 127;
  const int k = M - 2 - e;
  constexpr int L = (1 << (M - 1)) - 1;
  int q[kBlock];
#pragma unroll
  for (int t = 0; t < kBlock; ++t) {
    int c = __float2int_rn(scale_pow2(v[t], k));
    q[t] = min(max(c, -L), L);
  }
  *sdst = static_cast<uint8_t>(ef);
  if constexpr (M == 4) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t x = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) x |= (static_cast<uint32_t>(q[8 * j + i]) & 0xFu) << (4 * i);
      w[j] = x;
    }
    *reinterpret_cast<uint4 *>(cdst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (M == 6) {
    unsigned long long d[3] = {0ull, 0ull, 0ull};
#pragma unroll
    for (int t = 0; t < kBlock; ++t) {
      const unsigned long long f = static_cast<unsigned long long>(q[t] & 0x3F);
      const int pos = 6 * t, word = pos >> 6, off = pos & 63;
      d[word] |= f << off;
      if (off > 58) d[word + 1] |= f >> (64 - off);
    }
    unsigned long long *p = reinterpret_cast<unsigned long long *>(cdst);
    p[0] = d[0];
    p[1] = d[1];
    p[2] = d[2];
  } else {
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t x = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) x |= (static_cast<uint32_t>(q[4 * j + i]) & 0xFFu) << (8 * i);
      w[j] = x;
    }
    uint4 *p = reinterpret_cast<uint4 *>(cdst);
    p[0] = make_uint4(w[0], w[1], w[2], w[3]);
    p[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

template <bool F32>
__device__ __forceinline__ float load_elem(const void *base, int64_t idx) {
  if constexpr (F32) return __ldg(reinterpret_cast<const float *>(base) + idx);
  else return bf16_bits_to_float(__ldg(reinterpret_cast<const unsigned short *>(base) + idx));
}

template <bool F32>
__device__ __forceinline__ float smem_elem(const uint8_t *row, int64_t idx) {
  if constexpr (F32) return reinterpret_cast<const float *>(row)[idx];
  else return bf16_bits_to_float(reinterpret_cast<const unsigned short *>(row)[idx]);
}

__device__ __forceinline__ void locate_block(const QuantArgs &a, int blk, int &g, int &b) {
  if (blk < a.nb[0]) { g = 0; b = blk; }
  else if (blk < a.nb[0] + a.nb[1]) { g = 1; b = blk - a.nb[0]; }
  else { g = 2; b = blk - a.nb[0] - a.nb[1]; }
}

template <bool F32>
__device__ __forceinline__ void code_block(const QuantArgs &a, int64_t row, int g, int b,
                                           const float (&v)[kBlock]) {
  uint8_t *cdst = a.codes[g] + row * a.cpitch[g] + static_cast<int64_t>(b) * kBlock * seg_bits(g) / 8;
  uint8_t *sdst = a.scales[g] + row * a.spitch[g] + b;
  if (g == 0) encode_store<8>(v, cdst, sdst);
  else if (g == 1) encode_store<6>(v, cdst, sdst);
  else encode_store<4>(v, cdst, sdst);
}

// Flat grid over (row, block): positions read straight from global memory.
// Used for the identity layout (K/V cache) and when the staged path does not
// fit in shared memory.
template <bool F32>
__global__ void __launch_bounds__(256) quant_direct_kernel(QuantArgs a) {
  const int64_t total = a.rows * a.nb_total;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / a.nb_total;
    const int blk = static_cast<int>(i - row * a.nb_total);
    int g, b;
    locate_block(a, blk, g, b);
    const int64_t p0 = static_cast<int64_t>(b) * kBlock;
    const int64_t rbase = row * a.ld;
    float v[kBlock];
#pragma unroll
    for (int t = 0; t < kBlock; ++t) {
      const int64_t p = p0 + t;
      float x = 0.f;
      if (p < a.k_real[g]) {
        const int64_t col = a.perm ? __ldg(a.perm + a.real_off[g] + p) : a.real_off[g] + p;
        x = load_elem<F32>(a.src, rbase + col);
      }
      v[t] = x;
    }
    code_block<F32>(a, row, g, b, v);
  }
}

constexpr int kQuantThreads = 128;

__host__ __device__ inline int64_t perm_smem_words(int64_t K) { return (K / 32 + 1) * 33; }

// CTA per row (grid-stride): stage the permutation once and each row once in
// shared memory, then one thread per block gathers, codes and stores.
template <bool F32>
__global__ void __launch_bounds__(kQuantThreads) quant_staged_kernel(QuantArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  int32_t *sperm = reinterpret_cast<int32_t *>(smem);
  uint8_t *srow = smem + round_up(perm_smem_words(a.K) * 4, 16);
  constexpr int ES = F32 ? 4 : 2;
  for (int64_t i = threadIdx.x; i < a.K; i += blockDim.x)
    sperm[(i >> 5) * 33 + (i & 31)] = __ldg(a.perm + i);
  const int64_t row_bytes = a.K * ES;
  for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
    __syncthreads();
    const uint8_t *gsrc = reinterpret_cast<const uint8_t *>(a.src) + row * a.ld * ES;
    int64_t done = 0;
    if ((reinterpret_cast<uintptr_t>(gsrc) & 15u) == 0) {
      const int64_t n16 = row_bytes / 16;
      const uint4 *s16 = reinterpret_cast<const uint4 *>(gsrc);
      uint4 *d16 = reinterpret_cast<uint4 *>(srow);
      for (int64_t i = threadIdx.x; i < n16; i += blockDim.x) d16[i] = __ldg(s16 + i);
      done = n16 * 16;
    }
    for (int64_t i = done + threadIdx.x * ES; i < row_bytes; i += blockDim.x * ES) {
      if constexpr (F32) *reinterpret_cast<float *>(srow + i) = __ldg(reinterpret_cast<const float *>(gsrc + i));
      else *reinterpret_cast<unsigned short *>(srow + i) = __ldg(reinterpret_cast<const unsigned short *>(gsrc + i));
    }
    __syncthreads();
    for (int blk = threadIdx.x; blk < a.nb_total; blk += blockDim.x) {
      int g, b;
      locate_block(a, blk, g, b);
      const int64_t p0 = static_cast<int64_t>(b) * kBlock;
      float v[kBlock];
#pragma unroll
      for (int t = 0; t < kBlock; ++t) {
        const int64_t p = p0 + t;
        float x = 0.f;
        if (p < a.k_real[g]) {
          const int64_t r = a.real_off[g] + p;
          x = smem_elem<F32>(srow, sperm[(r >> 5) * 33 + (r & 31)]);
        }
        v[t] = x;
      }
      code_block<F32>(a, row, g, b, v);
    }
  }
}

// Decoder: one thread per block, values q * 2^(e - m + 2) written as fp32 in
// padded-position order.
struct DequantArgs {
  int64_t rows;
  int32_t nb[3];
  int32_t nb_total;
  int64_t k_off[3];
  const uint8_t *codes[3];
  int64_t cpitch[3];
  const uint8_t *scales[3];
  int64_t spitch[3];
  float *out;
  int64_t ldo;
};

__global__ void dequant_kernel(DequantArgs a) {
  const int64_t total = a.rows * a.nb_total;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / a.nb_total;
    int blk = static_cast<int>(i - row * a.nb_total);
    int g = 0;
    while (blk >= a.nb[g]) { blk -= a.nb[g]; ++g; }
    const int m = seg_bits(g);
    const uint8_t *c = a.codes[g] + row * a.cpitch[g] + static_cast<int64_t>(blk) * kBlock * m / 8;
    const int e = static_cast<int>(a.scales[g][row * a.spitch[g] + blk]) - 127;
    const float step = pow2f(e - m + 2);
    float *o = a.out + row * a.ldo + a.k_off[g] + static_cast<int64_t>(blk) * kBlock;
    for (int t = 0; t < kBlock; ++t) {
      int v;
      if (m == 8) {
        v = static_cast<int8_t>(c[t]);
      } else if (m == 4) {
        v = (c[t >> 1] >> (4 * (t & 1))) & 0xF;
        v = v >= 8 ? v - 16 : v;
      } else {
        const int grp = t >> 2, sub = t & 3;
        const uint32_t w = c[3 * grp] | (c[3 * grp + 1] << 8) | (c[3 * grp + 2] << 16);
        v = (w >> (6 * sub)) & 0x3F;
        v = v >= 32 ? v - 64 : v;
      }
      o[t] = static_cast<float>(v) * step;
    }
  }
}

}  // namespace mxs

using namespace mxs;

// ------------------------------------------------------------------ C ABI

extern "C" const char *mxs_status_str(mxs_status st) {
  switch (st) {
    case MXS_OK: return "MXS_OK";
    case MXS_ERR_ARG: return "MXS_ERR_ARG: bad argument";
    case MXS_ERR_SHAPE: return "MXS_ERR_SHAPE: inconsistent shapes or layouts";
    case MXS_ERR_ALIGN: return "MXS_ERR_ALIGN: pointer or pitch not 16-byte aligned";
    case MXS_ERR_DTYPE: return "MXS_ERR_DTYPE: unsupported element type";
    case MXS_ERR_BUDGET: return "MXS_ERR_BUDGET: the fixed 8-bit blocks exceed the budget";
    case MXS_ERR_CUDA: return "MXS_ERR_CUDA: CUDA runtime error";
    case MXS_ERR_TIMEOUT: return "MXS_ERR_TIMEOUT: a device-side bounded wait expired";
    case MXS_ERR_DEVICE: return "MXS_ERR_DEVICE: current device is not sm_100";
    case MXS_ERR_WORKSPACE: return "MXS_ERR_WORKSPACE: workspace missing, misaligned or too small";
  }
  return "unknown mxs_status";
}

extern "C" int64_t mxs_launch_count(void) {
  std::lock_guard<std::mutex> lk(g_launch_mu);
  return g_launches;
}

extern "C" mxs_status mxs_layout_make(int64_t K, const int64_t counts[3], const int32_t *perm,
                                      mxs_layout *out) {
  if (!counts || !out || K < 0) return MXS_ERR_ARG;
  int64_t sum = 0, off = 0;
  for (int g = 0; g < 3; ++g) {
    if (counts[g] < 0) return MXS_ERR_ARG;
    sum += counts[g];
  }
  if (sum != K) return MXS_ERR_SHAPE;
  out->K = K;
  out->perm = perm;
  for (int g = 0; g < 3; ++g) {
    out->seg[g].bits = kSegBits[g];
    out->seg[g].k_real = counts[g];
    out->seg[g].k_pad = pad32(counts[g]);
    out->seg[g].k_off = off;
    off += out->seg[g].k_pad;
  }
  out->K_pad = off;
  return MXS_OK;
}

extern "C" mxs_status mxs_mxtensor_bytes(int64_t rows, const mxs_layout *lay, int64_t code_pitch[3],
                                         int64_t code_bytes[3], int64_t scale_pitch[3],
                                         int64_t scale_bytes[3]) {
  if (rows < 0 || !code_pitch || !code_bytes || !scale_pitch || !scale_bytes) return MXS_ERR_ARG;
  mxs_status st = check_layout(lay);
  if (st != MXS_OK) return st;
  for (int g = 0; g < 3; ++g) {
    const mxs_segment &s = lay->seg[g];
    code_pitch[g] = s.k_pad ? round_up(seg_row_bytes(s.k_pad, s.bits), 16) : 0;
    scale_pitch[g] = s.k_pad ? round_up(s.k_pad / kBlock, 16) : 0;
    code_bytes[g] = rows * code_pitch[g];
    scale_bytes[g] = rows * scale_pitch[g];
  }
  return MXS_OK;
}

static mxs_status quantize_impl(const void *src, mxs_dtype dt, int64_t rows, int64_t ld,
                                const mxs_mxtensor *out, void *stream) {
  if (!out || !dtype_ok(dt)) return !out ? MXS_ERR_ARG : MXS_ERR_DTYPE;
  mxs_status st = check_mxtensor(out);
  if (st != MXS_OK) return st;
  if (rows != out->rows || ld < out->lay.K) return MXS_ERR_SHAPE;
  if (rows == 0 || out->lay.K_pad == 0) return MXS_OK;
  if (!src) return MXS_ERR_ARG;
  if ((st = check_device()) != MXS_OK) return st;

  QuantArgs a{};
  a.src = src;
  a.ld = ld;
  a.rows = rows;
  a.K = out->lay.K;
  a.perm = out->lay.perm;
  int64_t real = 0;
  a.nb_total = 0;
  for (int g = 0; g < 3; ++g) {
    const mxs_segment &s = out->lay.seg[g];
    a.k_real[g] = s.k_real;
    a.real_off[g] = real;
    real += s.k_real;
    a.nb[g] = static_cast<int32_t>(s.k_pad / kBlock);
    a.nb_total += a.nb[g];
    a.codes[g] = out->codes[g];
    a.cpitch[g] = out->code_pitch[g];
    a.scales[g] = out->scales[g];
    a.spitch[g] = out->scale_pitch[g];
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool f32 = dt == MXS_F32;
  const int64_t es = static_cast<int64_t>(dtype_size(dt));
  const int64_t smem = round_up(perm_smem_words(a.K) * 4, 16) + round_up(a.K * es, 16);
  const int nsm = sm_count();
  if (a.perm && smem <= 200 * 1024) {
    const int per_sm = std::max<int>(1, std::min<int>(16, static_cast<int>((220 * 1024) / (smem + 1024))));
    const int grid = static_cast<int>(std::min<int64_t>(rows, static_cast<int64_t>(nsm) * per_sm));
    if (f32) {
      cudaFuncSetAttribute(quant_staged_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      quant_staged_kernel<true><<<grid, kQuantThreads, smem, s>>>(a);
    } else {
      cudaFuncSetAttribute(quant_staged_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      quant_staged_kernel<false><<<grid, kQuantThreads, smem, s>>>(a);
    }
  } else {
    const int64_t total = rows * a.nb_total;
    const int grid = static_cast<int>(std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(nsm) * 8));
    if (f32) quant_direct_kernel<true><<<grid, 256, 0, s>>>(a);
    else quant_direct_kernel<false><<<grid, 256, 0, s>>>(a);
  }
  count_launch();
  return cuda_status(cudaGetLastError());
}

extern "C" mxs_status mxs_quantize_weight(const void *W, mxs_dtype dt, int64_t N, int64_t ldw,
                                          const mxs_mxtensor *out, void *stream) {
  return quantize_impl(W, dt, N, ldw, out, stream);
}

extern "C" mxs_status mxs_quantize_act(const void *A, mxs_dtype dt, int64_t M, int64_t lda,
                                       const mxs_mxtensor *out, void *stream) {
  return quantize_impl(A, dt, M, lda, out, stream);
}

extern "C" mxs_status mxs_dequantize(const mxs_mxtensor *in, float *out, int64_t ldo, void *stream) {
  mxs_status st = check_mxtensor(in);
  if (st != MXS_OK) return st;
  if (ldo < in->lay.K_pad) return MXS_ERR_SHAPE;
  if (in->rows == 0 || in->lay.K_pad == 0) return MXS_OK;
  if (!out) return MXS_ERR_ARG;
  if ((st = check_device()) != MXS_OK) return st;
  DequantArgs a{};
  a.rows = in->rows;
  a.nb_total = 0;
  for (int g = 0; g < 3; ++g) {
    a.nb[g] = static_cast<int32_t>(in->lay.seg[g].k_pad / kBlock);
    a.nb_total += a.nb[g];
    a.k_off[g] = in->lay.seg[g].k_off;
    a.codes[g] = in->codes[g];
    a.cpitch[g] = in->code_pitch[g];
    a.scales[g] = in->scales[g];
    a.spitch[g] = in->scale_pitch[g];
  }
  a.out = out;
  a.ldo = ldo;
  const int64_t total = a.rows * a.nb_total;
  const int grid = static_cast<int>(std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(sm_count()) * 8));
  dequant_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  count_launch();
  return cuda_status(cudaGetLastError());
}
