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

bool ensure_smem_impl(const void *kernel, int bytes) {
  struct Entry {
    const void *fn;
    int dev;
    int bytes;
  };
  static Entry table[256];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < used; ++i)
    if (table[i].fn == kernel && table[i].dev == dev && table[i].bytes >= bytes) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  for (int i = 0; i < used; ++i)
    if (table[i].fn == kernel && table[i].dev == dev) {
      table[i].bytes = bytes;
      return true;
    }
  if (used < 256) table[used++] = Entry{kernel, dev, bytes};
  return true;
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
  int64_t ld;            // elements
  int64_t rows;
  int32_t K;
  const int32_t *perm;   // NULL: identity
  int32_t k_real[3];
  int32_t real_off[3];   // first real position of each segment in perm order
  int32_t nb[3];         // blocks per row per segment
  int32_t nb_total;
  uint8_t *codes[3];
  int64_t cpitch[3];
  uint8_t *scales[3];
  int64_t spitch[3];
  int32_t rows_per_batch;  // rows staged per CTA iteration
  int32_t row_stride;      // staged row length in elements (>= K + 1, multiple of 8)
  int32_t vec_rows;        // rows are 16-byte aligned with K*esize % 16 == 0
};

constexpr uint32_t kMagic = 0x4B400000u;   // bits of 1.5 * 2^23: x + it rounds x to an integer, ties to even

// Codes one block: v[] holds the 32 values of the block in position order.
// The rounding uses the float unit: fma(v, 2^k, 1.5*2^23) rounds v*2^k (an
// exact product) to the nearest integer with ties to even, and the integer
// sits in the low mantissa bits of the result; clamping compares those bit
// patterns as unsigned integers.
template <int M>
__device__ __forceinline__ void encode_store(float (&v)[kBlock], uint8_t *cdst, uint8_t *sdst) {
  float amax = 0.f;
#pragma unroll
  for (int t = 0; t < kBlock; ++t) amax = fmaxf(amax, fabsf(v[t]));
  const int ef = static_cast<int>(__float_as_uint(amax) >> 23);   // E8M0 byte of the block
  int k = M - 2 - (ef == 0 ? -127 : ef - 127);
  if (k > 127) {                     // blocks below 2^-121: pre-scale by 2^64 (exact)
#pragma unroll
    for (int t = 0; t < kBlock; ++t) v[t] *= 18446744073709551616.0f;
    k -= 64;
  }
  const float sc = __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
  constexpr uint32_t L = (1u << (M - 1)) - 1u;
  uint32_t b[kBlock];
#pragma unroll
  for (int t = 0; t < kBlock; ++t) {
    uint32_t x = __float_as_uint(fmaf(v[t], sc, 12582912.0f));
    b[t] = min(max(x, kMagic - L), kMagic + L);
  }
  *sdst = static_cast<uint8_t>(ef);
  if constexpr (M == 4) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t x = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) x |= (b[8 * j + i] & 0xFu) << (4 * i);
      w[j] = x;
    }
    *reinterpret_cast<uint4 *>(cdst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (M == 6) {
    uint32_t w[6] = {0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
    for (int t = 0; t < kBlock; ++t) {
      const uint32_t f = b[t] & 0x3Fu;
      const int pos = 6 * t, word = pos >> 5, off = pos & 31;
      w[word] |= f << off;
      if (off > 26) w[word + 1] |= f >> (32 - off);
    }
    uint2 *q = reinterpret_cast<uint2 *>(cdst);
    q[0] = make_uint2(w[0], w[1]);
    q[1] = make_uint2(w[2], w[3]);
    q[2] = make_uint2(w[4], w[5]);
  } else {
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      w[j] = __byte_perm(__byte_perm(b[4 * j], b[4 * j + 1], 0x0040), __byte_perm(b[4 * j + 2], b[4 * j + 3], 0x0040),
                         0x5410);
    uint4 *q = reinterpret_cast<uint4 *>(cdst);
    q[0] = make_uint4(w[0], w[1], w[2], w[3]);
    q[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

template <bool F32>
__device__ __forceinline__ float staged_elem(const uint8_t *row, uint32_t idx) {
  if constexpr (F32) return reinterpret_cast<const float *>(row)[idx];
  else return bf16_bits_to_float(reinterpret_cast<const unsigned short *>(row)[idx]);
}

__device__ __forceinline__ void locate_block(const QuantArgs &a, int blk, int &g, int &b) {
  if (blk < a.nb[0]) { g = 0; b = blk; }
  else if (blk < a.nb[0] + a.nb[1]) { g = 1; b = blk - a.nb[0]; }
  else { g = 2; b = blk - a.nb[0] - a.nb[1]; }
}

__device__ __forceinline__ void code_block(const QuantArgs &a, int64_t row, int g, int b, float (&v)[kBlock]) {
  uint8_t *cdst = a.codes[g] + row * a.cpitch[g] + static_cast<int64_t>(b) * kBlock * seg_bits(g) / 8;
  uint8_t *sdst = a.scales[g] + row * a.spitch[g] + b;
  if (g == 0) encode_store<8>(v, cdst, sdst);
  else if (g == 1) encode_store<6>(v, cdst, sdst);
  else encode_store<4>(v, cdst, sdst);
}

constexpr int kQuantThreads = 256;
constexpr int kTabWordsPerBlock = 17;   // 32 uint16 source indices + 1 pad word: conflict-free pair reads

__host__ __device__ inline int64_t quant_table_bytes(int64_t nb_total) {
  return round_up(nb_total * kTabWordsPerBlock * 4, 16);
}

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Issues the copies of one batch of rows into a staging buffer (cp.async
// when rows are 16-byte aligned, plain loads otherwise).
template <bool F32>
__device__ __forceinline__ void stage_rows(const QuantArgs &a, int64_t r0, int nr, uint8_t *buf, int64_t srow_bytes) {
  constexpr int ES = F32 ? 4 : 2;
  if (a.vec_rows) {
    const int nvec = a.K * ES / 16;
    for (int i = threadIdx.x; i < nr * nvec; i += blockDim.x) {
      const int rr = i / nvec, v = i - rr * nvec;
      cp_async16(buf + rr * srow_bytes + v * 16,
                 reinterpret_cast<const uint8_t *>(a.src) + ((r0 + rr) * a.ld) * ES + v * 16);
    }
  } else {
    for (int i = threadIdx.x; i < nr * a.K; i += blockDim.x) {
      const int rr = i / a.K, c = i - rr * a.K;
      const int64_t gi = (r0 + rr) * a.ld + c;
      if constexpr (F32)
        reinterpret_cast<float *>(buf + rr * srow_bytes)[c] = __ldg(reinterpret_cast<const float *>(a.src) + gi);
      else
        reinterpret_cast<unsigned short *>(buf + rr * srow_bytes)[c] =
            __ldg(reinterpret_cast<const unsigned short *>(a.src) + gi);
    }
  }
}

// Persistent CTAs.  Prologue: the permutation is copied into shared memory
// (cp.async, all requests in flight) and turned into a gather table that maps
// every padded position of the layout to its source column (or to a zero
// slot past the row end), 32 uint16 entries per block in 17 words.  Loop:
// batches of rows stream through two staging buffers -- the copies of batch
// i+1 are in flight while one thread per block of batch i gathers its 32
// values through the table, codes and stores them.
template <bool F32>
__global__ void __launch_bounds__(kQuantThreads) quant_staged_kernel(QuantArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *tab = reinterpret_cast<uint32_t *>(smem);
  uint8_t *bufs = smem + quant_table_bytes(a.nb_total);
  constexpr int ES = F32 ? 4 : 2;
  const int RB = a.rows_per_batch;
  const int64_t srow_bytes = static_cast<int64_t>(a.row_stride) * ES;
  const int64_t buf_bytes = RB * srow_bytes;

  // prologue: permutation -> shared memory (the staging buffers are free yet)
  int32_t *sperm = reinterpret_cast<int32_t *>(bufs);
  if (a.perm) {
    if ((a.K & 3) == 0 && (reinterpret_cast<uintptr_t>(a.perm) & 15u) == 0) {
      for (int i = threadIdx.x; i < a.K / 4; i += blockDim.x) cp_async16(sperm + 4 * i, a.perm + 4 * i);
      cp_async_commit();
      cp_async_wait<0>();
    } else {
      for (int i = threadIdx.x; i < a.K; i += blockDim.x) sperm[i] = __ldg(a.perm + i);
    }
  }
  __syncthreads();
  unsigned short *tab16 = reinterpret_cast<unsigned short *>(tab);
  for (int i = threadIdx.x; i < a.nb_total * kBlock; i += blockDim.x) {
    const int blk = i >> 5, t = i & 31;
    int g, b;
    locate_block(a, blk, g, b);
    const int p = b * kBlock + t;
    int col = a.K;                                   // zero slot
    if (p < a.k_real[g]) col = a.perm ? sperm[a.real_off[g] + p] : a.real_off[g] + p;
    tab16[blk * (2 * kTabWordsPerBlock) + t] = static_cast<unsigned short>(col);
  }
  __syncthreads();
  for (int rr = threadIdx.x; rr < 2 * RB; rr += blockDim.x) {     // zero slots of both buffers
    if constexpr (F32) reinterpret_cast<float *>(bufs + rr * srow_bytes)[a.K] = 0.f;
    else reinterpret_cast<unsigned short *>(bufs + rr * srow_bytes)[a.K] = 0;
  }

  const int64_t nbatches = (a.rows + RB - 1) / RB;
  int64_t batch = blockIdx.x;
  if (batch < nbatches) stage_rows<F32>(a, batch * RB, static_cast<int>(min(static_cast<int64_t>(RB), a.rows - batch * RB)), bufs, srow_bytes);
  cp_async_commit();
  for (int it = 0; batch < nbatches; batch += gridDim.x, ++it) {
    const int64_t next = batch + gridDim.x;
    uint8_t *cur = bufs + (it & 1) * buf_bytes;
    if (next < nbatches)
      stage_rows<F32>(a, next * RB, static_cast<int>(min(static_cast<int64_t>(RB), a.rows - next * RB)),
                      bufs + ((it + 1) & 1) * buf_bytes, srow_bytes);
    cp_async_commit();
    cp_async_wait<1>();                              // the current batch has landed
    __syncthreads();
    const int64_t r0 = batch * RB;
    const int nr = static_cast<int>(min(static_cast<int64_t>(RB), a.rows - r0));
    const int items = nr * a.nb_total;
    for (int item = threadIdx.x; item < items; item += blockDim.x) {
      const int rr = item / a.nb_total, blk = item - rr * a.nb_total;
      int g, b;
      locate_block(a, blk, g, b);
      const uint32_t *tw = tab + blk * kTabWordsPerBlock;
      const uint8_t *srow = cur + rr * srow_bytes;
      float v[kBlock];
#pragma unroll
      for (int j = 0; j < kBlock / 2; ++j) {
        const uint32_t w = tw[j];
        v[2 * j] = staged_elem<F32>(srow, w & 0xFFFFu);
        v[2 * j + 1] = staged_elem<F32>(srow, w >> 16);
      }
      code_block(a, r0 + rr, g, b, v);
    }
    __syncthreads();                                 // buffer free for the copy issued next iteration
  }
  cp_async_wait<0>();
}

// Fallback when a staged row does not fit in shared memory (or K >= 65535):
// flat grid over (row, block), values read straight from global memory.
template <bool F32>
__global__ void __launch_bounds__(128) quant_direct_kernel(QuantArgs a) {
  const int64_t total = a.rows * a.nb_total;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / a.nb_total;
    const int blk = static_cast<int>(i - row * a.nb_total);
    int g, b;
    locate_block(a, blk, g, b);
    const int p0 = b * kBlock;
    const int64_t rbase = row * a.ld;
    float v[kBlock];
#pragma unroll
    for (int t = 0; t < kBlock; ++t) {
      const int p = p0 + t;
      float x = 0.f;
      if (p < a.k_real[g]) {
        const int64_t col = a.perm ? __ldg(a.perm + a.real_off[g] + p) : a.real_off[g] + p;
        if constexpr (F32) x = __ldg(reinterpret_cast<const float *>(a.src) + rbase + col);
        else x = bf16_bits_to_float(__ldg(reinterpret_cast<const unsigned short *>(a.src) + rbase + col));
      }
      v[t] = x;
    }
    code_block(a, row, g, b, v);
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
  if (rows != out->rows || ld < out->lay.K || out->lay.K > INT32_MAX / 2) return MXS_ERR_SHAPE;
  if (rows == 0 || out->lay.K_pad == 0) return MXS_OK;
  if (!src) return MXS_ERR_ARG;
  if ((st = check_device()) != MXS_OK) return st;

  QuantArgs a{};
  a.src = src;
  a.ld = ld;
  a.rows = rows;
  a.K = static_cast<int32_t>(out->lay.K);
  a.perm = out->lay.perm;
  int32_t real = 0;
  a.nb_total = 0;
  for (int g = 0; g < 3; ++g) {
    const mxs_segment &sg = out->lay.seg[g];
    a.k_real[g] = static_cast<int32_t>(sg.k_real);
    a.real_off[g] = real;
    real += static_cast<int32_t>(sg.k_real);
    a.nb[g] = static_cast<int32_t>(sg.k_pad / kBlock);
    a.nb_total += a.nb[g];
    a.codes[g] = out->codes[g];
    a.cpitch[g] = out->code_pitch[g];
    a.scales[g] = out->scales[g];
    a.spitch[g] = out->scale_pitch[g];
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool f32 = dt == MXS_F32;
  const int64_t es = static_cast<int64_t>(dtype_size(dt));
  a.row_stride = static_cast<int32_t>(round_up(a.K + 1, 8));
  a.vec_rows = aligned16(src) && (ld * es) % 16 == 0 && (a.K * es) % 16 == 0;
  const int64_t tab_bytes = quant_table_bytes(a.nb_total);
  const int64_t srow_bytes = a.row_stride * es;
  // rows per batch: about 16 KB of staged rows (two buffers), at least enough
  // blocks to occupy the CTA
  int64_t rb = std::max<int64_t>(1, (16 * 1024) / srow_bytes);
  rb = std::max<int64_t>(rb, (kQuantThreads + a.nb_total - 1) / a.nb_total);
  rb = std::min<int64_t>(rb, std::min<int64_t>(rows, 256));
  auto smem_of = [&](int64_t r) { return tab_bytes + std::max<int64_t>(2 * r * srow_bytes, round_up(a.K * 4, 16)); };
  int64_t smem = smem_of(rb);
  while (rb > 1 && smem > 160 * 1024) smem = smem_of(--rb);
  a.rows_per_batch = static_cast<int32_t>(rb);
  const int nsm = sm_count();
  const int64_t nbatch = (rows + rb - 1) / rb;
  const bool small = rows * a.nb_total <= 8192;       // prologue would dominate: read straight from global
  if (!small && a.K < 65535 && smem <= 200 * 1024) {
    const int per_sm = std::max<int>(1, std::min<int>(4, static_cast<int>((220 * 1024) / (smem + 1024))));
    const int grid = static_cast<int>(std::min<int64_t>(nbatch, static_cast<int64_t>(nsm) * per_sm));
    if (f32) {
      if (!ensure_smem(quant_staged_kernel<true>, 200 * 1024)) return MXS_ERR_CUDA;
      quant_staged_kernel<true><<<grid, kQuantThreads, smem, s>>>(a);
    } else {
      if (!ensure_smem(quant_staged_kernel<false>, 200 * 1024)) return MXS_ERR_CUDA;
      quant_staged_kernel<false><<<grid, kQuantThreads, smem, s>>>(a);
    }
  } else {
    const int64_t total = rows * a.nb_total;
    const int grid = static_cast<int>(std::min<int64_t>((total + 127) / 128, static_cast<int64_t>(nsm) * 16));
    if (f32) quant_direct_kernel<true><<<grid, 128, 0, s>>>(a);
    else quant_direct_kernel<false><<<grid, 128, 0, s>>>(a);
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
