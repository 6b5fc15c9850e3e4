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
// Kernel shapes.  (1) The tiled quantiser (a permuted layout): persistent
// CTAs, one per SM.  Batches of source rows stream into shared memory by
// bulk copies (TMA, three buffers in flight); each block's 32 values are
// gathered through a table built once per CTA from the permutation and coded
// by one thread.  A warp's unit of work is G rows x 32/G blocks of one
// segment (G = 8 when eight rows fit a buffer): lanes on different rows read
// the same table words (broadcast) and, with a row pitch of 16 bytes mod 128,
// mostly different banks for their gathers.  Warps take units from a shared
// counter with no CTA-wide barrier; the warp that finishes a batch's last
// unit refills its buffer.  (2) The identity layout (no permutation, e.g. the
// K/V cache): one thread per block, 16-byte loads straight from global
// memory.  (3) The lane quantiser, for a few rows or rows the bulk copies
// cannot take (unaligned pitch, rows too long to stage): one warp per block, one lane per
// position, the block maximum by a warp reduction and the packing by
// shuffles; its loads are all independent, so a tiny batch (a decode step)
// costs two memory latencies.
#include <algorithm>
#include <cstdio>
#include <mutex>

#include "mxs_internal.cuh"
#include "mxs_ptx.cuh"

namespace mxs {

static int64_t g_launches = 0;
static std::mutex g_launch_mu;

void count_launch(int n) {
  std::lock_guard<std::mutex> lk(g_launch_mu);
  g_launches += n;
}

unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext *);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long *);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

bool ensure_smem_impl(const void *kernel, int bytes) {
  struct Entry {
    const void *fn;
    unsigned long long ctx;
    int bytes;
  };
  static Entry table[256];
  static int used = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  unsigned long long ctx = current_context_id();
  if (ctx)
    for (int i = 0; i < used; ++i)
      if (table[i].fn == kernel && table[i].ctx == ctx && table[i].bytes >= bytes) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  ctx = current_context_id();   // the call above made the context current if it was not
  if (!ctx) return true;
  for (int i = 0; i < used; ++i)
    if (table[i].fn == kernel && table[i].ctx == ctx) {
      table[i].bytes = bytes;
      return true;
    }
  if (used < 256) table[used++] = Entry{kernel, ctx, bytes};
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
  int32_t boff[3];       // first block of each segment within a row
  uint32_t nb_magic[3];   // floor(2^32 / nb[g]) + 1: i / nb[g] == umulhi(i, magic) while i * nb[g] < 2^32
  int32_t rows_per_batch;  // rows staged per batch (a multiple of G)
  int32_t row_stride;      // staged row pitch in elements (> K, 16 bytes mod 128)
  int32_t lg;              // G = 1 << lg rows per work unit
  int32_t quads[3];        // units per G-row group in each segment (ceil(nb * G / 32))
  int32_t units_per_batch; // (rows_per_batch / G) * (quads[0] + quads[1] + quads[2])
};

// Maximum of |v[0..31]| (bit patterns of |x|, or of each 16-bit half),
// as a five-level tree: the chain of dependent max operations is 5 long.
__device__ __forceinline__ float absmax32(const float (&v)[kBlock]) {
  float m[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) m[i] = fmaxf(fabsf(v[i]), fabsf(v[i + 16]));
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
  return m[0];
}
// Packed bf16x2 magnitude max / min: max(|a|, |b|) or min(|a|, |b|) per
// half, carrying the XOR of the operands' signs (finite operands).
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t minabs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// Per half: the largest |x| over p[0..N-1], as bf16 bits with the sign clear.
template <int N>
__device__ __forceinline__ uint32_t absmax_u16x2(const uint32_t (&p)[N]) {
  uint32_t m[N / 2];
#pragma unroll
  for (int i = 0; i < N / 2; ++i) m[i] = maxabs_bf16x2(p[i], p[i + N / 2]);
#pragma unroll
  for (int w = N / 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = maxabs_bf16x2(m[i], m[i + w]);
  return m[0] & 0x7FFF7FFFu;
}
// bf16 bits of (2^(m-1) - 1) * 2^-k, the largest magnitude that codes
// below the clamp at width m (k in [-125, 128]).
template <int M>
__device__ __forceinline__ uint32_t clamp_bits(int k) {
  static_assert(M == 4 || M == 6, "packed path for 4- and 6-bit codes");
  return M == 4 ? (static_cast<uint32_t>(2 - k + 127) << 7) | 0x60u      // 7 = 1.75 * 2^2
                : (static_cast<uint32_t>(4 - k + 127) << 7) | 0x78u;     // 31 = 1.9375 * 2^4
}

constexpr uint32_t kMagic = 0x4B400000u;   // bits of 1.5 * 2^23: x + it rounds x to an integer, ties to even

// Codes one block: v[] holds the 32 values of the block in position order.
// The rounding uses the float unit: fma(v, 2^k, 1.5*2^23) rounds v*2^k (an
// exact product) to the nearest integer with ties to even, and the integer
// sits in the low mantissa bits of the result; clamping compares those bit
// patterns as unsigned integers.
template <int M>
__device__ __forceinline__ void encode_store(float (&v)[kBlock], uint8_t *cdst, uint8_t *sdst) {
  const float amax = absmax32(v);
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

// bf16 source, 4- and 6-bit codes: the same rule on packed pairs.  p[i]
// holds positions 2i (low half) and 2i+1 (high half) as bf16 bits.  The
// block maximum is a bf16x2 max of the magnitudes, so the E8M0 byte is its
// exponent field, as for fp32.  The clamp comes first, on the magnitude:
// |x| is cut to L * 2^-k (L = 2^(m-1) - 1, sign kept), which codes to the
// same integer as clamping after the rounding.  Rounding: one bf16x2 fma
// x*2^k + 192 (a single rounding of the exact value; 192 + q stays in
// [128, 256), where bf16 steps by 1) leaves the lane's bits at 0x4340 + q,
// and the code is the low m bits.  When k > 125 the block is tiny and takes the fp32
// path, so that subnormal inputs never reach the bf16 fma.
__device__ __forceinline__ uint32_t fma_bf16x2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

template <int M>
__device__ __forceinline__ void encode_store_bf16(const uint32_t (&p)[kBlock / 2], uint8_t *cdst, uint8_t *sdst) {
  static_assert(M == 4 || M == 6, "packed path for 4- and 6-bit codes");
  const uint32_t m2 = absmax_u16x2(p);
  const int ef = static_cast<int>(max(m2 & 0xFFFFu, m2 >> 16) >> 7);
  const int k = M - 2 - (ef == 0 ? -127 : ef - 127);
  if (k > 125) {
    float v[kBlock];
#pragma unroll
    for (int i = 0; i < kBlock / 2; ++i) {
      v[2 * i] = __uint_as_float(p[i] << 16);
      v[2 * i + 1] = __uint_as_float(p[i] & 0xFFFF0000u);
    }
    encode_store<M>(v, cdst, sdst);
    return;
  }
  const uint32_t sb = static_cast<uint32_t>(k + 127) << 7;
  const uint32_t s2 = sb | (sb << 16);
  const uint32_t cb = clamp_bits<M>(k);
  const uint32_t c2 = cb | (cb << 16);
  uint32_t r[kBlock / 2];
#pragma unroll
  for (int i = 0; i < kBlock / 2; ++i) r[i] = fma_bf16x2(minabs_bf16x2(p[i], c2), s2, 0x43404340u);
  *sdst = static_cast<uint8_t>(ef);
  if constexpr (M == 4) {
    // bytes of positions 4j..4j+3 (low byte of each lane), then each
    // byte's nibble joined with the next byte's: bytes 0 and 2 hold two codes
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t x = __byte_perm(r[4 * j], r[4 * j + 1], 0x6420);
      const uint32_t y = __byte_perm(r[4 * j + 2], r[4 * j + 3], 0x6420);
      const uint32_t zx = (x & 0x0F0F0F0Fu) | ((x >> 4) & 0xF0F0F0F0u);
      const uint32_t zy = (y & 0x0F0F0F0Fu) | ((y >> 4) & 0xF0F0F0F0u);
      w[j] = __byte_perm(zx, zy, 0x6420);
    }
    *reinterpret_cast<uint4 *>(cdst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    // 24-bit groups of four codes, then eight groups into six words
    uint32_t u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t x = __byte_perm(r[2 * j], r[2 * j + 1], 0x6420);
      const uint32_t z = (x & 0x003F003Fu) | ((x >> 2) & 0x0FC00FC0u);
      u[j] = (z & 0xFFFu) | ((z >> 4) & 0xFFF000u);
    }
    uint32_t w[6];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      w[3 * h] = u[4 * h] | (u[4 * h + 1] << 24);
      w[3 * h + 1] = (u[4 * h + 1] >> 8) | (u[4 * h + 2] << 16);
      w[3 * h + 2] = (u[4 * h + 2] >> 16) | (u[4 * h + 3] << 8);
    }
    uint2 *q = reinterpret_cast<uint2 *>(cdst);
    q[0] = make_uint2(w[0], w[1]);
    q[1] = make_uint2(w[2], w[3]);
    q[2] = make_uint2(w[4], w[5]);
  }
}

// Value at byte offset `off` of a staged row.
template <bool F32>
__device__ __forceinline__ float staged_elem(const uint8_t *row, uint32_t off) {
  if constexpr (F32) return *reinterpret_cast<const float *>(row + off);
  else return bf16_bits_to_float(*reinterpret_cast<const unsigned short *>(row + off));
}

__device__ __forceinline__ void locate_block(const QuantArgs &a, int blk, int &g, int &b) {
  if (blk < a.nb[0]) { g = 0; b = blk; }
  else if (blk < a.nb[0] + a.nb[1]) { g = 1; b = blk - a.nb[0]; }
  else { g = 2; b = blk - a.nb[0] - a.nb[1]; }
}

constexpr int kQuantThreads = 512;
constexpr int kQuantSmemBudget = 224 * 1024;   // per CTA (one CTA per SM)
constexpr int kQStages = 3;
// 32 byte offsets per block + 4 pad words: 16-byte reads of up to 8
// different blocks by one warp fall in different banks
constexpr int kTabWordsPerBlock = 36;
constexpr long long kQuantWaitLimit = 2000000000LL;   // cycles (~1 s)

__host__ __device__ inline int64_t quant_table_bytes(int64_t nb_total) {
  return round_up(nb_total * kTabWordsPerBlock * 4, 128);
}

// Warp-wide: issues the bulk copies of batch `batch` (one per row, rows
// spread over the lanes) into buffer `buf`, completing on `bar`.
template <bool F32>
__device__ __forceinline__ void issue_batch(const QuantArgs &a, int64_t batch, uint8_t *buf, int64_t srow_bytes,
                                            uint64_t *bar) {
  constexpr int ES = F32 ? 4 : 2;
  const int lane = threadIdx.x & 31;
  const int64_t r0 = batch * a.rows_per_batch;
  const int nr = static_cast<int>(min(static_cast<int64_t>(a.rows_per_batch), a.rows - r0));
  const uint32_t row_bytes = static_cast<uint32_t>(a.K) * ES;
  const uint8_t *src = reinterpret_cast<const uint8_t *>(a.src) + r0 * a.ld * ES;
  // the buffer's previous contents were read through the generic proxy
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (lane == 0) ptx::mbar_arrive_expect_tx(bar, row_bytes * nr);
  __syncwarp();
  for (int rr = lane; rr < nr; rr += 32) ptx::bulk_load(buf + rr * srow_bytes, src + rr * a.ld * ES, row_bytes, bar);
}

// Byte offsets in a staged row of positions 4j .. 4j+3 of block b of segment
// g: from the gather table in shared memory (TAB), else from the permutation
// itself (rows too wide for the table beside the staging buffers; the
// permutation stays in L2).  Positions past the segment's real columns read
// the zero slot at column K.
template <bool TAB, int ES>
__device__ __forceinline__ uint4 gather4(const QuantArgs &a, int g, int b, const uint32_t *tab, int j) {
  if constexpr (TAB) {
    return reinterpret_cast<const uint4 *>(tab + (a.boff[g] + b) * kTabWordsPerBlock)[j];
  } else {
    const int p0 = kBlock * b + 4 * j;
    if (a.perm && p0 + 3 < a.k_real[g]) {
      const int32_t *src = a.perm + a.real_off[g] + p0;
      if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
        const int4 v = __ldg(reinterpret_cast<const int4 *>(src));    // four real columns, one load
        return make_uint4(static_cast<uint32_t>(v.x * ES), static_cast<uint32_t>(v.y * ES),
                          static_cast<uint32_t>(v.z * ES), static_cast<uint32_t>(v.w * ES));
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int p = p0 + u;
      const int col = p < a.k_real[g] ? (a.perm ? __ldg(a.perm + a.real_off[g] + p) : a.real_off[g] + p) : a.K;
      o[u] = static_cast<uint32_t>(col * ES);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// One lane's item of a work unit: gathers block b of segment g (width M) of
// staged row `srow` and codes it into row `row`.
template <int M, bool F32, bool TAB>
__device__ __forceinline__ void code_item(const QuantArgs &a, int g, int b, const uint32_t *tab, const uint8_t *srow,
                                          int64_t row) {
  constexpr int ES = F32 ? 4 : 2;
  if constexpr (!F32 && M != 8) {
    uint32_t p[kBlock / 2];
#pragma unroll
    for (int j = 0; j < kBlock / 4; ++j) {
      const uint4 w = gather4<TAB, ES>(a, g, b, tab, j);
      p[2 * j] = static_cast<uint32_t>(*reinterpret_cast<const unsigned short *>(srow + w.x)) |
                 (static_cast<uint32_t>(*reinterpret_cast<const unsigned short *>(srow + w.y)) << 16);
      p[2 * j + 1] = static_cast<uint32_t>(*reinterpret_cast<const unsigned short *>(srow + w.z)) |
                     (static_cast<uint32_t>(*reinterpret_cast<const unsigned short *>(srow + w.w)) << 16);
    }
    encode_store_bf16<M>(p, a.codes[g] + row * a.cpitch[g] + b * (kBlock * M / 8), a.scales[g] + row * a.spitch[g] + b);
  } else {
    float v[kBlock];
#pragma unroll
    for (int j = 0; j < kBlock / 4; ++j) {
      const uint4 w = gather4<TAB, ES>(a, g, b, tab, j);
      v[4 * j] = staged_elem<F32>(srow, w.x);
      v[4 * j + 1] = staged_elem<F32>(srow, w.y);
      v[4 * j + 2] = staged_elem<F32>(srow, w.z);
      v[4 * j + 3] = staged_elem<F32>(srow, w.w);
    }
    encode_store<M>(v, a.codes[g] + row * a.cpitch[g] + b * (kBlock * M / 8), a.scales[g] + row * a.spitch[g] + b);
  }
}

// Polls with a growing sleep between reads, so that waiting warps leave the
// issue slots to the warps that are coding.
__device__ __forceinline__ bool spin_until_equal(volatile int *p, int want, long long limit) {
  if (*p == want) return true;
  const long long t0 = clock64();
  unsigned ns = 32;
  while (*p != want) {
    if (clock64() - t0 > limit) return false;
    __nanosleep(ns);
    ns = min(ns * 2, 512u);
  }
  return true;
}

// Persistent CTAs over their batches (local batch i = global batch
// blockIdx.x + i * gridDim.x, in buffer i mod kQStages).  Prologue: warp 0
// issues the first kQStages batches; meanwhile the CTA builds the gather
// table (every padded position of the layout -> its source column, or a zero
// slot past the row end, as byte offsets; 36 words per block) and writes
// the zero slots.  Loop (per warp): take the next unit, wait until its batch
// has been issued and has landed, code it, and count it done; the warp that
// completes a batch refills that buffer with the batch kQStages ahead.
template <bool F32, bool TAB>
__global__ void __launch_bounds__(kQuantThreads, 1) quant_tile_kernel(QuantArgs a, int *status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int ES = F32 ? 4 : 2;
  uint32_t *tab = reinterpret_cast<uint32_t *>(smem);
  const int64_t tab_bytes = TAB ? quant_table_bytes(a.nb_total) : 0;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + tab_bytes);
  uint8_t *bufs = smem + tab_bytes + 128;
  __shared__ int next_unit, abort_flag;
  __shared__ int done_cnt[kQStages];
  __shared__ int issued[kQStages];
  const int lane = threadIdx.x & 31;
  const int RB = a.rows_per_batch;
  const int64_t srow_bytes = static_cast<int64_t>(a.row_stride) * ES;
  const int64_t buf_bytes = RB * srow_bytes;
  const int64_t nbatches = (a.rows + RB - 1) / RB;
  const int nloc = blockIdx.x < nbatches ? static_cast<int>((nbatches - blockIdx.x + gridDim.x - 1) / gridDim.x) : 0;

  if (threadIdx.x == 0) {
    next_unit = 0;
    abort_flag = 0;
#pragma unroll
    for (int st = 0; st < kQStages; ++st) {
      ptx::mbar_init(&bar[st], 1);
      done_cnt[st] = 0;
      issued[st] = -1;
    }
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    for (int st = 0; st < kQStages && st < nloc; ++st)
      issue_batch<F32>(a, blockIdx.x + static_cast<int64_t>(st) * gridDim.x, bufs + st * buf_bytes, srow_bytes,
                       &bar[st]);
    __syncwarp();
    if (lane == 0)
      for (int st = 0; st < kQStages; ++st) issued[st] = st < nloc ? st : -1;   // -1: never copied into
  }
  // gather table: 8 permutation loads in flight per thread
  for (int g = 0; TAB && g < 3; ++g) {
    const int n = a.nb[g] * kBlock;
    for (int p0 = threadIdx.x; p0 < n; p0 += 8 * kQuantThreads) {
      int col[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int p = p0 + u * kQuantThreads;
        col[u] = a.K;                                  // zero slot
        if (p < a.k_real[g]) col[u] = a.perm ? __ldg(a.perm + a.real_off[g] + p) : a.real_off[g] + p;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int p = p0 + u * kQuantThreads;
        if (p < n) tab[(a.boff[g] + (p >> 5)) * kTabWordsPerBlock + (p & 31)] = static_cast<uint32_t>(col[u] * ES);
      }
    }
  }
  for (int rr = threadIdx.x; rr < kQStages * RB; rr += kQuantThreads) {   // zero slots (never copied over)
    if constexpr (F32) reinterpret_cast<float *>(bufs + rr * srow_bytes)[a.K] = 0.f;
    else reinterpret_cast<unsigned short *>(bufs + rr * srow_bytes)[a.K] = 0;
  }
  __syncthreads();

  const int ups = a.units_per_batch;
  const int qt = a.quads[0] + a.quads[1] + a.quads[2];
  const int G = 1 << a.lg;
  const int total = nloc * ups;
  for (;;) {
    int u = 0;
    if (lane == 0) u = atomicAdd(&next_unit, 1);
    u = __shfl_sync(0xffffffffu, u, 0);
    if (u >= total || *reinterpret_cast<volatile int *>(&abort_flag)) break;
    const int it = u / ups, ul = u - it * ups;
    const int st = it % kQStages;
    bool ok = spin_until_equal(&issued[st], it, kQuantWaitLimit);
    ok = ok && ptx::mbar_wait_cycles(&bar[st], (it / kQStages) & 1, kQuantWaitLimit);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) {
        abort_flag = 1;
        atomicExch(status, static_cast<int>(MXS_ERR_TIMEOUT));
      }
      break;
    }
    // unit -> (row group, segment, quad); lane -> (row in group, block of quad)
    const int rg = ul / qt;
    int q = ul - rg * qt, g = 0;
    if (q >= a.quads[0]) {
      q -= a.quads[0];
      g = 1;
      if (q >= a.quads[1]) {
        q -= a.quads[1];
        g = 2;
      }
    }
    const int64_t r0 = (blockIdx.x + static_cast<int64_t>(it) * gridDim.x) * RB;
    const int rl = rg * G + (lane & (G - 1));
    const int b = q * (32 >> a.lg) + (lane >> a.lg);
    if (r0 + rl < a.rows && b < a.nb[g]) {
      const uint8_t *srow = bufs + st * buf_bytes + rl * srow_bytes;
      if (g == 0) code_item<8, F32, TAB>(a, 0, b, tab, srow, r0 + rl);
      else if (g == 1) code_item<6, F32, TAB>(a, 1, b, tab, srow, r0 + rl);
      else code_item<4, F32, TAB>(a, 2, b, tab, srow, r0 + rl);
    }
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&done_cnt[st], 1) == ups - 1;
    }
    if (__shfl_sync(0xffffffffu, last, 0)) {
      // every unit of batch it is done: its buffer is free
      if (lane == 0) done_cnt[st] = 0;
      const int nx = it + kQStages;
      if (nx < nloc) {
        issue_batch<F32>(a, blockIdx.x + static_cast<int64_t>(nx) * gridDim.x, bufs + st * buf_bytes, srow_bytes,
                         &bar[st]);
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          atomicExch(&issued[st], nx);
        }
      }
    }
  }
  __syncthreads();
  if (abort_flag && threadIdx.x == 0) {
    // let copies still in flight land (bounded) before the shared memory is released
    for (int st = 0; st < kQStages; ++st) {
      const int it = issued[st];
      if (it >= 0) ptx::mbar_wait_cycles(&bar[st], (it / kQStages) & 1, kQuantWaitLimit);
    }
  }
}

// ------------------------------------------- transposed quantiser (bf16)
//
// For bf16 sources with a permuted layout.  A batch is 8 source rows, bulk
// copied (one copy per row) into a row-major buffer.  Four transposer warps
// turn it, 8 x 8 at a time (ldmatrix .trans, stmatrix), into a copy T in
// which each column of the batch is 16 contiguous bytes: rows 2p and 2p+1
// form 32-bit word p.  The coding warps then gather a block's 32 positions
// for two rows with one 32-bit load each and code both rows at once in
// packed bf16 pairs (one row per half).  T is double-buffered, so the
// transposers fill the next batch while the coders drain this one; coders
// take 32-lane units (4 row pairs x 8 blocks of one segment) from a shared
// counter.  Within a segment the layout keeps the columns in ascending
// order, so in a dense segment the 8 blocks of a unit read columns 32
// apart; T therefore stores column c in slot c ^ ((c >> 3 ^ c >> 6) & 7) of
// its 8-column group, which spreads such strides over the banks.  Hand-off: monotone
// counters in shared memory, the transposers publishing the batch a buffer
// holds and the coders counting finished units per buffer.

constexpr int kTrRows = 8;                 // rows per batch
constexpr int kTrThreads = 640;
constexpr int kTrTransposers = 4;          // warps 0..3

struct TrArgs {
  QuantArgs q;
  int32_t kc;             // columns of T holding data (K rounded up to 32); column kc is zero
  int32_t nt;             // T buffers (1 or 2)
  int32_t pitch;          // bytes per staged source row (16 mod 128)
  int32_t units[3];       // coding units per batch in each segment
  int32_t U;              // units per batch
  uint32_t U_magic;       // floor(2^32 / U) + 1 (0 when U == 1)
  int32_t t_off, raw_off, tab_off;   // shared-memory layout (bytes)
};

// T slot of column c (a bijection within each aligned group of 8 columns).
__host__ __device__ inline int32_t tr_slot(int32_t c) { return (c & ~7) | ((c ^ (c >> 3) ^ (c >> 6)) & 7); }
__host__ __device__ inline int64_t tr_t_bytes(int64_t kc) { return (kc + 8) * 16; }

// Both rows of a T word pair (low half: row 2p, high half: row 2p+1) coded
// at width M into their own rows.  Per row the rule is that of
// encode_store_bf16; rows whose block is tiny take the fp32 coder.
template <int M>
__device__ __forceinline__ void encode2_store(const uint32_t (&v)[kBlock], uint8_t *c0, uint8_t *s0, uint8_t *c1,
                                              uint8_t *s1, bool has1) {
  const uint32_t m2 = absmax_u16x2(v);
  const int ef0 = static_cast<int>((m2 & 0xFFFFu) >> 7), ef1 = static_cast<int>(m2 >> 23);
  const int k0 = M - 2 - (ef0 == 0 ? -127 : ef0 - 127), k1 = M - 2 - (ef1 == 0 ? -127 : ef1 - 127);
  if (M == 8 || k0 > 125 || k1 > 125) {
    float x[kBlock];
#pragma unroll
    for (int t = 0; t < kBlock; ++t) x[t] = __uint_as_float(v[t] << 16);
    encode_store<M>(x, c0, s0);
    if (has1) {
#pragma unroll
      for (int t = 0; t < kBlock; ++t) x[t] = __uint_as_float(v[t] & 0xFFFF0000u);
      encode_store<M>(x, c1, s1);
    }
    return;
  }
  if constexpr (M != 8) {
    const uint32_t s2 = (static_cast<uint32_t>(k0 + 127) << 7) | (static_cast<uint32_t>(k1 + 127) << 23);
    const uint32_t c2 = clamp_bits<M>(k0) | (clamp_bits<M>(k1) << 16);
    uint32_t r[kBlock];
#pragma unroll
    for (int t = 0; t < kBlock; ++t) r[t] = fma_bf16x2(minabs_bf16x2(v[t], c2), s2, 0x43404340u);
    *s0 = static_cast<uint8_t>(ef0);
    if (has1) *s1 = static_cast<uint8_t>(ef1);
    if constexpr (M == 4) {
      // a lane's low nibble is the code (0x40 + q).  Word pair (r[2i], r[2i+1])
      // -> t: byte 0 = row 0's codes of positions 2i, 2i+1 (low nibble first),
      // byte 2 = row 1's, by one select of r[2i]'s low nibbles against
      // r[2i+1] shifted up a nibble; bytes 1 and 3 are never read
      uint32_t w0[4], w1[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t t[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t a = r[8 * j + 2 * k], b = r[8 * j + 2 * k + 1] << 4;
          t[k] = (a & 0x000F000Fu) | (b & 0xFFF0FFF0u);
        }
        const uint32_t u0 = __byte_perm(t[0], t[1], 0x6240), u1 = __byte_perm(t[2], t[3], 0x6240);
        w0[j] = __byte_perm(u0, u1, 0x5410);      // row 0, positions 8j .. 8j+7
        w1[j] = __byte_perm(u0, u1, 0x7632);      // row 1
      }
      *reinterpret_cast<uint4 *>(c0) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
      if (has1) *reinterpret_cast<uint4 *>(c1) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
    } else {
      // x0[j] / x1[j]: the low bytes of positions 4j..4j+3 of row 0 / row 1
      uint32_t x0[8], x1[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t A = __byte_perm(r[4 * j], r[4 * j + 1], 0x6240);
        const uint32_t B = __byte_perm(r[4 * j + 2], r[4 * j + 3], 0x6240);
        x0[j] = __byte_perm(A, B, 0x5410);
        x1[j] = __byte_perm(A, B, 0x7632);
      }
      uint32_t u0[8], u1[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t z0 = (x0[j] & 0x003F003Fu) | ((x0[j] >> 2) & 0x0FC00FC0u);
        u0[j] = (z0 & 0xFFFu) | ((z0 >> 4) & 0xFFF000u);
        const uint32_t z1 = (x1[j] & 0x003F003Fu) | ((x1[j] >> 2) & 0x0FC00FC0u);
        u1[j] = (z1 & 0xFFFu) | ((z1 >> 4) & 0xFFF000u);
      }
      uint32_t w0[6], w1[6];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        w0[3 * h] = u0[4 * h] | (u0[4 * h + 1] << 24);
        w0[3 * h + 1] = (u0[4 * h + 1] >> 8) | (u0[4 * h + 2] << 16);
        w0[3 * h + 2] = (u0[4 * h + 2] >> 16) | (u0[4 * h + 3] << 8);
        w1[3 * h] = u1[4 * h] | (u1[4 * h + 1] << 24);
        w1[3 * h + 1] = (u1[4 * h + 1] >> 8) | (u1[4 * h + 2] << 16);
        w1[3 * h + 2] = (u1[4 * h + 2] >> 16) | (u1[4 * h + 3] << 8);
      }
      uint2 *q0 = reinterpret_cast<uint2 *>(c0);
      q0[0] = make_uint2(w0[0], w0[1]);
      q0[1] = make_uint2(w0[2], w0[3]);
      q0[2] = make_uint2(w0[4], w0[5]);
      if (has1) {
        uint2 *q1 = reinterpret_cast<uint2 *>(c1);
        q1[0] = make_uint2(w1[0], w1[1]);
        q1[1] = make_uint2(w1[2], w1[3]);
        q1[2] = make_uint2(w1[4], w1[5]);
      }
    }
  }
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ bool mbar_test_wait(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(ptx::smem_addr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void stsm_x4(uint32_t addr, const uint32_t (&r)[4]) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

// Bounded poll of a shared counter until it reaches `want` (monotone).
__device__ __forceinline__ bool spin_until_at_least(volatile int *p, int want, long long limit) {
  if (*p >= want) return true;
  const long long t0 = clock64();
  unsigned ns = 32;
  while (*p < want) {
    if (clock64() - t0 > limit) return false;
    __nanosleep(ns);
    ns = min(ns * 2, 256u);
  }
  return true;
}

// All-or-nothing decision of the transposer warps: every thread of the
// 128 passes its flag; every thread returns the OR.
__device__ __forceinline__ bool transposers_any(bool f) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(f))
      : "memory");
  return r != 0;
}

// Warp-wide: bulk-copies the rows of local batch i into the staging
// buffer, one row per lane, completing on `bar`.  The buffer's previous
// batch was read into registers and written to T before the transposers'
// barrier that precedes this call, so the copies overwrite nothing that is
// still to be read.
__device__ __forceinline__ void tr_issue_batch(const TrArgs &ta, int i, int nloc, uint8_t *raw, uint64_t *bar) {
  const QuantArgs &a = ta.q;
  const int lane = threadIdx.x & 31;
  const int64_t r0 = (blockIdx.x + static_cast<int64_t>(i) * gridDim.x) * kTrRows;
  const int nr = static_cast<int>(min(static_cast<int64_t>(kTrRows), a.rows - r0));
  const uint32_t bytes = static_cast<uint32_t>(a.K) * 2;
  const uint8_t *src = reinterpret_cast<const uint8_t *>(a.src);
  if (lane == 0) ptx::mbar_arrive_expect_tx(bar, bytes * nr);
  __syncwarp();
  if (lane < nr) ptx::bulk_load(raw + lane * ta.pitch, src + (r0 + lane) * a.ld * 2, bytes, bar);
  // the batch after: into L2 now, so that its copies wait on L2 only
  if (i + 1 < nloc) {
    const int64_t r1 = r0 + static_cast<int64_t>(gridDim.x) * kTrRows;
    if (lane < kTrRows && r1 + lane < a.rows)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src + (r1 + lane) * a.ld * 2), "r"(bytes)
                   : "memory");
  }
}

__global__ void __launch_bounds__(kTrThreads, 1) quant_tr_kernel(TrArgs ta, int *status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  const QuantArgs &a = ta.q;
  uint32_t *tab = reinterpret_cast<uint32_t *>(smem + ta.tab_off);
  uint8_t *tbuf = smem + ta.t_off;
  uint8_t *raw = smem + ta.raw_off;
  __shared__ __align__(8) uint64_t raw_full;
  __shared__ int next_unit, abort_flag;
  __shared__ int ready[2], done[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nbatches = (a.rows + kTrRows - 1) / kTrRows;
  const int nloc = blockIdx.x < nbatches ? static_cast<int>((nbatches - blockIdx.x + gridDim.x - 1) / gridDim.x) : 0;
  const int64_t tbytes = round_up(tr_t_bytes(ta.kc), 128);
  volatile int *vabort = &abort_flag;

  if (threadIdx.x == 0) {
    next_unit = 0;
    abort_flag = 0;
    ready[0] = ready[1] = -1;
    done[0] = done[1] = 0;
    ptx::mbar_init(&raw_full, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0 && nloc > 0) tr_issue_batch(ta, 0, nloc, raw, &raw_full);
  // gather table: T byte offset (slot * 16) of each layout position's
  // column, the zero column for padding; every position's permutation load
  // is independent, 8 in flight per thread
  const int npos = a.nb_total * kBlock;
  for (int p0 = threadIdx.x; p0 < npos; p0 += 8 * kTrThreads) {
    int col[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int pa = p0 + u * kTrThreads;
      const int g = pa < a.boff[1] * kBlock ? 0 : (pa < a.boff[2] * kBlock ? 1 : 2);
      const int p = pa - a.boff[g] * kBlock;
      col[u] = ta.kc;
      if (pa < npos && p < a.k_real[g]) col[u] = __ldg(a.perm + a.real_off[g] + p);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int pa = p0 + u * kTrThreads;
      if (pa < npos) tab[(pa >> 5) * kTabWordsPerBlock + (pa & 31)] = static_cast<uint32_t>(tr_slot(col[u])) * 16u;
    }
  }
  if (threadIdx.x < ta.nt)
    *reinterpret_cast<uint4 *>(tbuf + threadIdx.x * tbytes + tr_slot(ta.kc) * 16) = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();

  if (warp < kTrTransposers) {
    const int ngroups = ta.kc / 32;
    const int m = lane >> 3, r = lane & 7;
    const uint32_t raw_row = ptx::smem_addr(raw + r * ta.pitch + 16 * m);
    int inflight = nloc > 0 ? 0 : -1;                 // batch whose rows are being copied
    for (int i = 0; i < nloc; ++i) {
      const int s = ta.nt == 2 ? (i & 1) : 0;
      const uint32_t T = ptx::smem_addr(tbuf + s * tbytes) + 128 * m;
      // T[s] is free once every unit of the batches it held is done; the
      // batch's rows have landed
      bool bad = false;
      // (one thread waits; the others take the completed phase after the
      // barrier, which a non-blocking test then observes at once)
      if (threadIdx.x == 0)
        bad = !spin_until_at_least(&done[s], (ta.nt == 2 ? (i >> 1) : i) * ta.U, kQuantWaitLimit) ||
              !ptx::mbar_wait_cycles(&raw_full, i & 1, kQuantWaitLimit);
      if (transposers_any(bad || *vabort)) {
        if (threadIdx.x == 0) *vabort = 1;
        break;
      }
      if (threadIdx.x != 0 && !mbar_test_wait(&raw_full, i & 1)) ptx::mbar_wait_cycles(&raw_full, i & 1, kQuantWaitLimit);
      inflight = -1;
      __threadfence_block();
      for (int g0 = warp; g0 < ngroups; g0 += 4 * kTrTransposers) {
        uint32_t v[4][4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int gi = g0 + k * kTrTransposers;
          if (gi < ngroups) ldsm_x4_trans(raw_row + gi * 64, v[k]);
        }
        // stmatrix writes row r of matrix m, i.e. T column c = 32 gi + 8 m + r,
        // at the address this lane gives: the slot keeps the group (c & ~7)
        // and XORs the low 3 bits with (c >> 3 ^ c >> 6)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int gi = g0 + k * kTrTransposers;
          if (gi < ngroups) {
            const uint32_t h = static_cast<uint32_t>((4 * gi + m) ^ (gi >> 1)) & 7u;
            stsm_x4(T + static_cast<uint32_t>(gi) * 512 + ((static_cast<uint32_t>(r) ^ h) << 4), v[k]);
          }
        }
      }
      // every transposer is done: the batch is published and the staging
      // buffer takes the next batch
      transposers_any(false);
      if (threadIdx.x == 0) {
        __threadfence_block();
        *reinterpret_cast<volatile int *>(&ready[s]) = i;
      }
      if (i + 1 < nloc) {
        if (warp == 0) tr_issue_batch(ta, i + 1, nloc, raw, &raw_full);
        inflight = i + 1;
      }
    }
    // an aborted run leaves no bulk copy in flight
    if (threadIdx.x == 0 && inflight >= 0) ptx::mbar_wait_cycles(&raw_full, inflight & 1, kQuantWaitLimit);
  } else {
    const int total = nloc * ta.U;
    for (;;) {
      int v = 0;
      if (lane == 0) v = atomicAdd(&next_unit, 1);
      v = __shfl_sync(0xffffffffu, v, 0);
      if (v >= total || *vabort) break;
      const int i = ta.U == 1 ? v : static_cast<int>(__umulhi(static_cast<uint32_t>(v), ta.U_magic));
      const int u = v - i * ta.U;
      const int s = ta.nt == 2 ? (i & 1) : 0;
      int ok = 1;
      if (lane == 0) {
        const long long t0 = clock64();
        unsigned ns = 32;
        while (*reinterpret_cast<volatile int *>(&ready[s]) < i) {
          if (*vabort || clock64() - t0 > kQuantWaitLimit) {
            ok = 0;
            break;
          }
          __nanosleep(ns);
          ns = min(ns * 2, 64u);
        }
        __threadfence_block();
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) *vabort = 1;
        break;
      }
      int g = 0, qd = u;
      if (qd >= ta.units[0]) {
        qd -= ta.units[0];
        g = 1;
        if (qd >= ta.units[1]) {
          qd -= ta.units[1];
          g = 2;
        }
      }
      const int pr = lane & 3, bb = qd * 8 + (lane >> 2);
      const int64_t r0 = (blockIdx.x + static_cast<int64_t>(i) * gridDim.x) * kTrRows + 2 * pr;
      if (bb < a.nb[g] && r0 < a.rows) {
        const uint32_t T = ptx::smem_addr(tbuf + s * tbytes) + pr * 4;
        const uint32_t tw = ptx::smem_addr(tab + (a.boff[g] + bb) * kTabWordsPerBlock);
        uint32_t x[kBlock];
#pragma unroll
        for (int j = 0; j < kBlock / 4; ++j) {
          const uint4 w = lds128(tw + 16 * j);
          x[4 * j] = lds32(T + w.x);
          x[4 * j + 1] = lds32(T + w.y);
          x[4 * j + 2] = lds32(T + w.z);
          x[4 * j + 3] = lds32(T + w.w);
        }
        const bool has1 = r0 + 1 < a.rows;
        uint8_t *s0 = a.scales[g] + r0 * a.spitch[g] + bb;
        if (g == 0) {
          uint8_t *c0 = a.codes[0] + r0 * a.cpitch[0] + bb * 32;
          encode2_store<8>(x, c0, s0, c0 + a.cpitch[0], s0 + a.spitch[0], has1);
        } else if (g == 1) {
          uint8_t *c0 = a.codes[1] + r0 * a.cpitch[1] + bb * 24;
          encode2_store<6>(x, c0, s0, c0 + a.cpitch[1], s0 + a.spitch[1], has1);
        } else {
          uint8_t *c0 = a.codes[2] + r0 * a.cpitch[2] + bb * 16;
          encode2_store<4>(x, c0, s0, c0 + a.cpitch[2], s0 + a.spitch[2], has1);
        }
      }
      // every lane's reads of T are done before the unit counts as finished
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        atomicAdd(&done[s], 1);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *vabort) atomicExch(status, static_cast<int>(MXS_ERR_TIMEOUT));
}

// Identity layout: one thread per (row, block), values read straight from
// global memory (16-byte loads when the block's 32 source values are
// aligned and all real).
template <bool F32>
__global__ void __launch_bounds__(256) quant_contig_kernel(QuantArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int ES = F32 ? 4 : 2;
  const int64_t total = a.rows * a.nb_total;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / a.nb_total;
    const int blk = static_cast<int>(i - row * a.nb_total);
    int g, b;
    locate_block(a, blk, g, b);
    const int p0 = b * kBlock;
    const int64_t e0 = row * a.ld + a.real_off[g] + p0;       // element index of position p0
    const int n = min(kBlock, a.k_real[g] - p0);
    float v[kBlock];
    const uint8_t *base = reinterpret_cast<const uint8_t *>(a.src) + e0 * ES;
    uint8_t *cdst = a.codes[g] + row * a.cpitch[g] + static_cast<int64_t>(b) * kBlock * seg_bits(g) / 8;
    uint8_t *sdst = a.scales[g] + row * a.spitch[g] + b;
    if (!F32 && g != 0 && n == kBlock && (reinterpret_cast<uintptr_t>(base) & 15u) == 0) {
      uint32_t p[kBlock / 2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(base) + j);
        p[4 * j] = x.x;
        p[4 * j + 1] = x.y;
        p[4 * j + 2] = x.z;
        p[4 * j + 3] = x.w;
      }
      if (g == 1) encode_store_bf16<6>(p, cdst, sdst);
      else encode_store_bf16<4>(p, cdst, sdst);
      continue;
    }
    if (n == kBlock && (reinterpret_cast<uintptr_t>(base) & 15u) == 0) {
#pragma unroll
      for (int j = 0; j < kBlock * ES / 16; ++j) {
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(base) + j);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if constexpr (F32) {
            v[4 * j + k] = __uint_as_float(w[k]);
          } else {
            v[8 * j + 2 * k] = __uint_as_float(w[k] << 16);
            v[8 * j + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
          }
        }
      }
    } else {
#pragma unroll
      for (int t = 0; t < kBlock; ++t) {
        float x = 0.f;
        if (t < n) {
          if constexpr (F32) x = __ldg(reinterpret_cast<const float *>(a.src) + e0 + t);
          else x = bf16_bits_to_float(__ldg(reinterpret_cast<const unsigned short *>(a.src) + e0 + t));
        }
        v[t] = x;
      }
    }
    if (g == 0) encode_store<8>(v, cdst, sdst);
    else if (g == 1) encode_store<6>(v, cdst, sdst);
    else encode_store<4>(v, cdst, sdst);
  }
}

// The K/V cache layout {0, 0, K} (one 4-bit segment, no permutation) on
// bf16 rows of K % 32 == 0 values: one thread per 32-value block, its 64
// source bytes read by two 32-byte loads, coded by encode_store_bf16's rule
// and stored as one 16-byte code word and one scale byte.  Block i of the
// tensor is row i / nb, block i % nb (a 32-bit multiply-high division); each
// thread takes kKvU blocks, their loads issued together.
constexpr int kKvU = 2;
constexpr int kKvThreads = 128;

__device__ __forceinline__ void ld_stream_32B(const void *p, uint32_t (&w)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
               : "l"(p));
}

__global__ void __launch_bounds__(kKvThreads) quant_kv4_kernel(QuantArgs a, uint32_t total) {
  pdl_wait();
  pdl_trigger();
  const uint32_t nb = static_cast<uint32_t>(a.nb[2]);
  const uint32_t stride = gridDim.x * blockDim.x;
  const uint16_t *src = static_cast<const uint16_t *>(a.src);
  for (uint32_t i0 = blockIdx.x * blockDim.x + threadIdx.x; i0 < total; i0 += kKvU * stride) {
    uint32_t p[kKvU][16], row[kKvU], b[kKvU];
#pragma unroll
    for (int u = 0; u < kKvU; ++u) {
      const uint32_t i = i0 + u * stride;
      row[u] = nb > 1 ? __umulhi(i, a.nb_magic[2]) : i;
      b[u] = i - row[u] * nb;
      if (i < total) {
        const uint16_t *blk = src + static_cast<int64_t>(row[u]) * a.ld + b[u] * kBlock;
        uint32_t lo[8], hi[8];
        ld_stream_32B(blk, lo);
        ld_stream_32B(blk + 16, hi);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          p[u][t] = lo[t];
          p[u][8 + t] = hi[t];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kKvU; ++u) {
      if (i0 + u * stride >= total) break;
      encode_store_bf16<4>(p[u], a.codes[2] + static_cast<int64_t>(row[u]) * a.cpitch[2] + b[u] * 16,
                           a.scales[2] + static_cast<int64_t>(row[u]) * a.spitch[2] + b[u]);
    }
  }
}

// One warp per (row, block), one lane per position.
template <bool F32>
__global__ void __launch_bounds__(256) quant_lane_kernel(QuantArgs a) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t total = a.rows * a.nb_total;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total; w += nwarps) {
    const int64_t row = w / a.nb_total;
    const int blk = static_cast<int>(w - row * a.nb_total);
    int g, b;
    locate_block(a, blk, g, b);
    const int m = seg_bits(g);
    const int p = b * kBlock + lane;
    float x = 0.f;
    if (p < a.k_real[g]) {
      const int64_t col = a.perm ? __ldg(a.perm + a.real_off[g] + p) : a.real_off[g] + p;
      if constexpr (F32) x = __ldg(reinterpret_cast<const float *>(a.src) + row * a.ld + col);
      else x = bf16_bits_to_float(__ldg(reinterpret_cast<const unsigned short *>(a.src) + row * a.ld + col));
    }
    const uint32_t ab = __reduce_max_sync(0xffffffffu, __float_as_uint(x) & 0x7FFFFFFFu);
    const int ef = static_cast<int>(ab >> 23);
    int k = m - 2 - (ef == 0 ? -127 : ef - 127);
    if (k > 127) {                     // blocks below 2^-121: pre-scale by 2^64 (exact)
      x *= 18446744073709551616.0f;
      k -= 64;
    }
    const uint32_t L = (1u << (m - 1)) - 1u;
    uint32_t q = __float_as_uint(fmaf(x, __uint_as_float(static_cast<uint32_t>(k + 127) << 23), 12582912.0f));
    q = min(max(q, kMagic - L), kMagic + L);         // low m bits: the two's-complement code
    uint8_t *cdst = a.codes[g] + row * a.cpitch[g] + static_cast<int64_t>(b) * kBlock * m / 8;
    const uint32_t q1 = __shfl_down_sync(0xffffffffu, q, 1);
    const uint32_t q2 = __shfl_down_sync(0xffffffffu, q, 2);
    const uint32_t q3 = __shfl_down_sync(0xffffffffu, q, 3);
    if (m == 8) {
      cdst[lane] = static_cast<uint8_t>(q);
    } else if (m == 4) {
      if ((lane & 1) == 0) cdst[lane >> 1] = static_cast<uint8_t>((q & 0xFu) | ((q1 & 0xFu) << 4));
    } else if ((lane & 3) == 0) {
      const uint32_t w24 = (q & 63u) | ((q1 & 63u) << 6) | ((q2 & 63u) << 12) | ((q3 & 63u) << 18);
      uint8_t *d = cdst + (lane >> 2) * 3;
      d[0] = static_cast<uint8_t>(w24);
      d[1] = static_cast<uint8_t>(w24 >> 8);
      d[2] = static_cast<uint8_t>(w24 >> 16);
    }
    if (lane == 0) a.scales[g][row * a.spitch[g] + b] = static_cast<uint8_t>(ef);
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
  pdl_wait();
  pdl_trigger();
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
  int32_t boff = 0;
  for (int g = 0; g < 3; ++g) {
    a.boff[g] = boff;
    boff += a.nb[g];
    // (nb == 1 divides trivially and has no 32-bit magic)
    a.nb_magic[g] = a.nb[g] > 1 ? static_cast<uint32_t>((1ull << 32) / static_cast<uint64_t>(a.nb[g]) + 1) : 0u;
  }
  const int nsm = sm_count();
  const int64_t warps = rows * a.nb_total;
  const bool tiny = warps <= 8192;                     // latency-bound: one warp per block
  if (!tiny && !a.perm && !f32 && a.k_real[0] == 0 && a.k_real[1] == 0 && a.K % kBlock == 0 && aligned16(src) &&
      (ld * 2) % 32 == 0 && (reinterpret_cast<uintptr_t>(src) & 31u) == 0 && warps < (1ll << 31) &&
      (a.nb[2] <= 1 || warps * a.nb[2] < (1ll << 32))) {
    // the K/V cache: one 4-bit segment, rows of whole blocks (32-byte
    // aligned); 128-thread CTAs, so that the SMs' shares differ by at most
    // one small CTA
    const int grid = static_cast<int>(std::min<int64_t>((warps + kKvThreads * kKvU - 1) / (kKvThreads * kKvU),
                                                        static_cast<int64_t>(nsm) * 16));
    launch_pdl(quant_kv4_kernel, dim3(grid), dim3(kKvThreads), 0, s, a, static_cast<uint32_t>(warps));
    count_launch();
    return cuda_status(cudaGetLastError());
  }
  if (!tiny && !a.perm) {
    const int grid = static_cast<int>(std::min<int64_t>((warps + 255) / 256, static_cast<int64_t>(nsm) * 8));
    if (f32) launch_pdl(quant_contig_kernel<true>, dim3(grid), dim3(256), 0, s, a);
    else launch_pdl(quant_contig_kernel<false>, dim3(grid), dim3(256), 0, s, a);
    count_launch();
    return cuda_status(cudaGetLastError());
  }
  // staged paths: rows bulk-copyable (16-byte aligned base, pitch and row
  // length) and small enough to stage
  const bool vec_rows = aligned16(src) && (ld * es) % 16 == 0 && (a.K * es) % 16 == 0;
  if (!tiny && vec_rows && !f32) {
    // transposed path when two column-major copies of a batch, its staged
    // rows and the gather table fit
    TrArgs ta{};
    ta.kc = static_cast<int32_t>(round_up(a.K, 32));
    ta.pitch = static_cast<int32_t>(round_up(static_cast<int64_t>(a.K) * 2, 128) + 16);
    const int64_t tb = round_up(tr_t_bytes(ta.kc), 128);
    const int64_t tab = quant_table_bytes(a.nb_total);
    const int64_t rawb = round_up(static_cast<int64_t>(kTrRows) * ta.pitch, 128);
    ta.nt = tab + 2 * tb + rawb <= kQuantSmemBudget ? 2 : 0;
    if (ta.nt > 0) {
      ta.q = a;
      ta.U = 0;
      for (int g = 0; g < 3; ++g) {
        ta.units[g] = (a.nb[g] + 7) / 8;
        ta.U += ta.units[g];
      }
      ta.U_magic = ta.U > 1 ? static_cast<uint32_t>((1ull << 32) / static_cast<uint64_t>(ta.U) + 1) : 0u;
      ta.tab_off = 0;
      ta.t_off = static_cast<int32_t>(tab);
      ta.raw_off = static_cast<int32_t>(tab + ta.nt * tb);
      const int64_t tsmem = ta.raw_off + rawb;
      const int64_t nbatches = (rows + kTrRows - 1) / kTrRows;
      const int tgrid = static_cast<int>(std::min<int64_t>(nsm, nbatches));
      int *status = device_status_word();
      if (!status) return MXS_ERR_CUDA;
      if (!ensure_smem(quant_tr_kernel, static_cast<int>(tsmem))) return MXS_ERR_CUDA;
      launch_pdl(quant_tr_kernel, dim3(tgrid), dim3(kTrThreads), tsmem, s, ta, status);
      count_launch();
      return cuda_status(cudaGetLastError());
    }
  }
  bool tiled = !tiny && vec_rows;
  bool tab = true;            // gather table in shared memory, else offsets from the permutation
  int64_t smem = 0;
  int grid = 0;
  if (tiled) {
    // pitch: room for the zero slot, 16 bytes mod 128
    const int64_t pitch = round_up((a.K + 1) * es, 128) + 16;
    a.row_stride = static_cast<int32_t>(pitch / es);
    int64_t fixed = quant_table_bytes(a.nb_total) + 128;
    int64_t rows_fit = std::min<int64_t>(256, (kQuantSmemBudget - fixed) / kQStages / pitch);
    if (rows_fit < 1) {
      // rows too wide for the table beside three row buffers (K above about
      // 20 K for bf16): stage the rows alone and read the permutation from L2
      tab = false;
      fixed = 128;
      rows_fit = std::min<int64_t>(256, (kQuantSmemBudget - fixed) / kQStages / pitch);
    }
    tiled = rows_fit >= 1;
    if (tiled) {
      a.lg = rows_fit >= 8 ? 3 : rows_fit >= 4 ? 2 : rows_fit >= 2 ? 1 : 0;
      const int64_t G = 1 << a.lg;
      // rows per batch: a multiple of G, every CTA about the same number of batches
      const int64_t rb_max = rows_fit / G * G;
      const int64_t rounds = (rows + nsm * rb_max - 1) / (nsm * rb_max);
      const int64_t rb = std::min(rb_max, round_up((rows + nsm * rounds - 1) / (nsm * rounds), G));
      a.rows_per_batch = static_cast<int32_t>(rb);
      int32_t qsum = 0;
      for (int g = 0; g < 3; ++g) {
        a.quads[g] = static_cast<int32_t>((a.nb[g] * G + 31) / 32);
        qsum += a.quads[g];
      }
      a.units_per_batch = static_cast<int32_t>(rb / G) * qsum;
      grid = static_cast<int>(std::min<int64_t>(nsm, (rows + rb - 1) / rb));
      smem = fixed + kQStages * rb * pitch;
    }
  }
  if (tiled) {
    int *status = device_status_word();
    if (!status) return MXS_ERR_CUDA;
    auto go = [&](auto kernel) -> mxs_status {
      if (!ensure_smem(kernel, static_cast<int>(smem))) return MXS_ERR_CUDA;
      launch_pdl(kernel, dim3(grid), dim3(kQuantThreads), smem, s, a, status);
      return MXS_OK;
    };
    const mxs_status st = f32 ? (tab ? go(quant_tile_kernel<true, true>) : go(quant_tile_kernel<true, false>))
                              : (tab ? go(quant_tile_kernel<false, true>) : go(quant_tile_kernel<false, false>));
    if (st != MXS_OK) return st;
  } else {
    const int lgrid = static_cast<int>(std::min<int64_t>((warps + 7) / 8, static_cast<int64_t>(nsm) * 16));
    if (f32) launch_pdl(quant_lane_kernel<true>, dim3(lgrid), dim3(256), 0, s, a);
    else launch_pdl(quant_lane_kernel<false>, dim3(lgrid), dim3(256), 0, s, a);
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
  launch_pdl(dequant_kernel, dim3(grid), dim3(256), 0, reinterpret_cast<cudaStream_t>(stream), a);
  count_launch();
  return cuda_status(cudaGetLastError());
}
