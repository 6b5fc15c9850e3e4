// mxs_decode.cu -- mxs_gemm for a handful of activation rows (decode).
//
// MXSens (arXiv 2607.17733), technical summary §2.3 and §4: the mixed
// 4/6/8-bit MXINT linear layer; at decode the product is bound by the bytes
// of the packed weights, which this path reads once.
#include <algorithm>

#include "mxs_decode.cuh"
#include "mxs_ptx.cuh"

namespace mxs {

// ------------------------------------------------------ small-M decode path
//
// For a handful of activation rows the GEMM is bound by the bytes of W, so
// W is read packed, once, and never expanded in memory.  Within one
// 32-position block both operands share one E8M0 scale each, so the block's
// contribution is an integer dot product times an exact power of two:
//   sum_t qa_t qw_t * 2^(ea - m + 2) * 2^(ew - m + 2).
// Every code is widened to a signed byte holding code * 2^(8-m) (the code
// in the top bits of the byte: a mask, no sign extension), so one 32-column
// block of either operand is 32 int8 values and the block's integer dot
// product is exactly one tensor-core mma.sync m16n8k32 (s8 x s8 -> s32),
// 16 activation rows x 8 W rows.  |sum| < 2^22, so the int32 converts
// exactly, and the scale 2^(ea-6) * 2^(ew-6) is exact; only the fp32
// accumulation over blocks (and the final bf16 rounding) rounds.  The block
// scaling forbids accumulating across blocks inside the tensor core, which
// is why the block-sized warp-level MMA is used here rather than tcgen05.
//
// Each CTA owns 16 W rows (two n-tiles of 8); its eight warps split the K
// blocks of each segment (warp w takes blocks w, w+8, ...).  One warp
// bulk-copies (TMA) the activations' packed code and scale rows and the 16 W
// rows' packed code and scale rows into shared memory, so every byte the CTA
// needs is in flight at once; every lane then builds, per block, its A and
// B fragments from the shared copies, widening only the two 4-code groups a
// fragment holds.  When the W rows do not fit beside the activations, their
// codes stream from global memory instead (through L1, several blocks in
// flight).  The warps' partial sums are added in shared memory in warp
// order.  Calls whose packed activation rows do not fit in shared memory
// take the tensor-core path.
struct SmallArgs {
  int32_t M, N;
  int32_t nb[3];
  int32_t nb_total;
  const uint8_t *a_codes[3];
  int64_t a_cpitch[3];
  const uint8_t *a_scales[3];
  int64_t a_spitch[3];
  const uint8_t *w_codes[3];
  int64_t w_cpitch[3];
  const uint8_t *w_scales[3];
  int64_t w_spitch[3];
  __nv_bfloat16 *Y;
  int64_t ldy;
  int32_t stage_w;       // the W rows' codes are copied into shared memory too
};

constexpr int kDecRows = 16;                 // W rows per CTA (two n-tiles of 8)
constexpr int kDecMaxM = 16;                 // activation rows: the MMA's 16 rows
constexpr int kDecWarps = 8;                 // K slots
constexpr int kDecThreads = kDecWarps * 32;

__device__ __forceinline__ void small_locate(const SmallArgs &a, int gb, int &g, int &b) {
  if (gb < a.nb[0]) { g = 0; b = gb; }
  else if (gb < a.nb[0] + a.nb[1]) { g = 1; b = gb - a.nb[0]; }
  else { g = 2; b = gb - a.nb[0] - a.nb[1]; }
}

// Four 4-bit codes (16 bits, code i in nibble i) -> four bytes code << 4.
__device__ __forceinline__ uint32_t widen4(uint32_t x16) {
  const uint32_t p = __byte_perm(x16, 0, 0x1100);       // bytes b0 b0 b1 b1
  return ((p << 4) & 0x00F000F0u) | (p & 0xF000F000u);
}
// Four 6-bit codes (24 bits, code i at bits 6i) -> four bytes code << 2.
__device__ __forceinline__ uint32_t widen6(uint32_t v) {
  return ((v << 2) & 0xFCu) | ((v << 4) & 0xFC00u) | ((v << 6) & 0xFC0000u) | ((v << 8) & 0xFC000000u);
}

__device__ __forceinline__ void mma_s8_16x8x32(const uint4 &a, uint32_t b0, uint32_t b1, int (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1), "r"(0), "r"(0), "r"(0), "r"(0));
}

// A W word read from global memory through L1: the four lanes of a block
// row and the warps on neighbouring blocks share its 32-byte sectors, which
// L1 then serves once instead of L2 four times.
__device__ __forceinline__ uint32_t ld_stream_u32(const uint8_t *p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// Per segment: raw words one lane loads for its B fragment of one W block,
// and how many blocks a warp keeps in flight.
template <int G> struct DecSeg;
template <> struct DecSeg<0> { static constexpr int kRaw = 2, kU = 4; };   // 8-bit: words t, 4+t
template <> struct DecSeg<1> { static constexpr int kRaw = 2, kU = 4; };   // 6-bit: one word pair, codes 8t..8t+7
template <> struct DecSeg<2> { static constexpr int kRaw = 1, kU = 8; };   // 4-bit: one word, codes 8t..8t+7

__device__ __forceinline__ uint32_t lds_u32(const uint8_t *p) { return *reinterpret_cast<const uint32_t *>(p); }

// The words of block c (packed, m-bit) that lane-in-group t needs for its
// fragment: code groups t and 4+t (codes 4t..4t+3 and 16+4t..16+4t+3) for
// 8-bit blocks; for 6- and 4-bit blocks, codes 8t..8t+7 (one word pair, one
// word), which fill the same fragment slots in another order.  A and W take
// the same order, so every code still meets its partner and the integer dot
// product is unchanged.
// SMEM: c points into shared memory (activations), else into global memory
// (W, streaming loads).
template <int G, bool SMEM>
__device__ __forceinline__ void load_frag_raw(const uint8_t *c, int t, uint32_t (&r)[DecSeg<G>::kRaw]) {
  if constexpr (G == 2) {
    r[0] = SMEM ? lds_u32(c + 4 * t) : ld_stream_u32(c + 4 * t);
  } else if constexpr (G == 0) {
    r[0] = SMEM ? lds_u32(c + 4 * t) : ld_stream_u32(c + 4 * t);
    r[1] = SMEM ? lds_u32(c + 16 + 4 * t) : ld_stream_u32(c + 16 + 4 * t);
  } else {
    // codes 8t..8t+7: bytes 6t..6t+5, inside the two words from 4 floor(6t/4)
    const int w0 = (6 * t) & ~3;
    r[0] = SMEM ? lds_u32(c + w0) : ld_stream_u32(c + w0);
    r[1] = SMEM ? lds_u32(c + w0 + 4) : ld_stream_u32(c + w0 + 4);
  }
}

template <int G>
__device__ __forceinline__ void widen_frag(const uint32_t (&r)[DecSeg<G>::kRaw], int t, uint32_t &b0, uint32_t &b1) {
  if constexpr (G == 2) {
    b0 = widen4(r[0] & 0xFFFFu);            // slots 4t..4t+3: codes 8t..8t+3
    b1 = widen4(r[0] >> 16);                // slots 16+4t..16+4t+3: codes 8t+4..8t+7
  } else if constexpr (G == 0) {
    b0 = r[0];
    b1 = r[1];
  } else {
    // the 48 bits of codes 8t..8t+7 start 0 or 16 bits into the pair
    const uint64_t v = ((static_cast<uint64_t>(r[1]) << 32) | r[0]) >> ((6 * t & 3) * 8);
    b0 = widen6(static_cast<uint32_t>(v));          // slots 4t..: codes 8t..8t+3 (low 24 bits)
    b1 = widen6(static_cast<uint32_t>(v >> 24));    // slots 16+4t..: codes 8t+4..8t+7
  }
}

// Shared-memory image of one CTA: per segment g, the activations' packed
// code rows (M rows at the source pitch), their scale rows, the scale rows
// of the CTA's 16 W rows (rows past N repeat row N-1) and, when they fit,
// the 16 W rows' packed codes, so that every byte the CTA reads is in
// flight from its first instruction.
struct DecSmem {
  int32_t a_code[3], a_scale[3], w_scale[3], w_code[3];
  int32_t bytes;
};

__host__ __device__ inline DecSmem dec_smem_plan(const SmallArgs &a) {
  DecSmem p{};
  int32_t off = 0;
  for (int g = 0; g < 3; ++g) {
    p.a_code[g] = off;
    off += a.nb[g] ? static_cast<int32_t>(a.M * a.a_cpitch[g]) : 0;
  }
  for (int g = 0; g < 3; ++g) {
    p.a_scale[g] = off;
    off += a.nb[g] ? static_cast<int32_t>(a.M * a.a_spitch[g]) : 0;
  }
  for (int g = 0; g < 3; ++g) {
    p.w_scale[g] = off;
    off += a.nb[g] ? static_cast<int32_t>(kDecRows * a.w_spitch[g]) : 0;
  }
  for (int g = 0; g < 3; ++g) {
    p.w_code[g] = off;
    off += a.stage_w && a.nb[g] ? static_cast<int32_t>(kDecRows * a.w_cpitch[g]) : 0;
  }
  p.bytes = off;
  return p;
}

// The blocks of segment G: warp w takes every 8th, kU per round with their
// W loads in flight together.
template <int G, bool SW>
__device__ __forceinline__ void dec_segment(const SmallArgs &a, const uint8_t *smem, const DecSmem &sp, int n0,
                                            float (&acc)[2][4]) {
  constexpr int MB = G == 0 ? 8 : (G == 1 ? 6 : 4);
  constexpr int BB = kBlock * MB / 8;                 // bytes per packed block
  constexpr int U = DecSeg<G>::kU, R = DecSeg<G>::kRaw;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int nbg = a.nb[G];
  const uint8_t *wc = a.w_codes[G];
  // this lane's rows: W rows n0 + 8j + gid (loads), activation rows gid, gid + 8
  const uint8_t *wrow[2];
#pragma unroll
  for (int j = 0; j < 2; ++j)
    wrow[j] = SW ? smem + sp.w_code[G] + (8 * j + gid) * a.w_cpitch[G]
                 : wc + static_cast<int64_t>(min(n0 + 8 * j + gid, a.N - 1)) * a.w_cpitch[G];
  const bool a_lo = gid < a.M, a_hi = gid + 8 < a.M;   // rows past M read as zero
  const uint8_t *arow_lo = smem + sp.a_code[G] + (a_lo ? gid : 0) * a.a_cpitch[G];
  const uint8_t *arow_hi = smem + sp.a_code[G] + (a_hi ? gid + 8 : 0) * a.a_cpitch[G];
  const uint8_t *asc = smem + sp.a_scale[G];
  const uint8_t *wsc = smem + sp.w_scale[G];
  for (int b0 = warp; b0 < nbg; b0 += kDecWarps * U) {
    uint32_t raw[U][2][R];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int bb = b0 + kDecWarps * u;
      if (bb < nbg) {
#pragma unroll
        for (int j = 0; j < 2; ++j) load_frag_raw<G, SW>(wrow[j] + bb * BB, tig, raw[u][j]);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int bb = b0 + kDecWarps * u;
      if (bb >= nbg) continue;
      // A fragment: rows gid / gid+8, code groups tig / 4+tig
      uint32_t ar[2][R];
      load_frag_raw<G, true>(arow_lo + bb * BB, tig, ar[0]);
      load_frag_raw<G, true>(arow_hi + bb * BB, tig, ar[1]);
      uint4 af;
      widen_frag<G>(ar[0], tig, af.x, af.z);
      widen_frag<G>(ar[1], tig, af.y, af.w);
      if (!a_lo) af.x = af.z = 0u;
      if (!a_hi) af.y = af.w = 0u;
      // bytes hold code * 2^(8-m): scale 2^(e-m+2) * 2^(m-8) = 2^(e-6)
      const float fa_lo = pow2f(static_cast<int>(asc[(a_lo ? gid : 0) * a.a_spitch[G] + bb]) - 127 - 6);
      const float fa_hi = pow2f(static_cast<int>(asc[(a_hi ? gid + 8 : 0) * a.a_spitch[G] + bb]) - 127 - 6);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        uint32_t f0, f1;
        widen_frag<G>(raw[u][j], tig, f0, f1);
        int c[4];
        mma_s8_16x8x32(af, f0, f1, c);
        const float fw0 = pow2f(static_cast<int>(wsc[(8 * j + 2 * tig) * a.w_spitch[G] + bb]) - 127 - 6);
        const float fw1 = pow2f(static_cast<int>(wsc[(8 * j + 2 * tig + 1) * a.w_spitch[G] + bb]) - 127 - 6);
        acc[j][0] = fmaf(code_to_float(c[0]), fa_lo * fw0, acc[j][0]);
        acc[j][1] = fmaf(code_to_float(c[1]), fa_lo * fw1, acc[j][1]);
        acc[j][2] = fmaf(code_to_float(c[2]), fa_hi * fw0, acc[j][2]);
        acc[j][3] = fmaf(code_to_float(c[3]), fa_hi * fw1, acc[j][3]);
      }
    }
  }
}

constexpr long long kDecWaitLimit = 2000000000LL;    // cycles (~1 s)

// One CTA: W rows n0 .. n0+15.  Rows of a packed segment lie at a fixed
// pitch, so the activations' code rows, their scale rows and the CTA's W
// scale (and, when staged, code) rows are each one contiguous range: one
// thread bulk-copies them into shared memory with one copy per range (a
// dozen copies, not one per row, which the copy engine would take one by
// one); W rows past N are not copied and only feed outputs that are never
// stored.  The copies complete on two barriers: the scale rows with the 8-
// and 6-bit codes, then the 4-bit codes, so the warps run the 8- and 6-bit
// segments while the 4-bit codes are still landing.  Then they add their
// partial sums in warp order.
__global__ void __launch_bounds__(kDecThreads) gemm_small_kernel(SmallArgs a, int *status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bar[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int n0 = blockIdx.x * kDecRows;
  const DecSmem sp = dec_smem_plan(a);
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar[0], 1);
    ptx::mbar_init(&bar[1], 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int wrows = min(kDecRows, a.N - n0);        // W rows of this CTA that exist
    uint32_t bytes[2] = {0u, 0u};
    for (int g = 0; g < 3; ++g) {
      if (!a.nb[g]) continue;
      bytes[0] += static_cast<uint32_t>(a.M * a.a_spitch[g] + wrows * a.w_spitch[g]);
      bytes[g == 2] += static_cast<uint32_t>(a.M * a.a_cpitch[g] + (a.stage_w ? wrows * a.w_cpitch[g] : 0));
    }
    ptx::mbar_arrive_expect_tx(&bar[0], bytes[0]);
    ptx::mbar_arrive_expect_tx(&bar[1], bytes[1]);
    for (int g = 0; g < 3; ++g) {
      if (!a.nb[g]) continue;
      uint64_t *cb = &bar[g == 2];
      ptx::bulk_load(smem + sp.a_scale[g], a.a_scales[g], static_cast<uint32_t>(a.M * a.a_spitch[g]), &bar[0]);
      ptx::bulk_load(smem + sp.w_scale[g], a.w_scales[g] + static_cast<int64_t>(n0) * a.w_spitch[g],
                     static_cast<uint32_t>(wrows * a.w_spitch[g]), &bar[0]);
      ptx::bulk_load(smem + sp.a_code[g], a.a_codes[g], static_cast<uint32_t>(a.M * a.a_cpitch[g]), cb);
      if (a.stage_w)
        ptx::bulk_load(smem + sp.w_code[g], a.w_codes[g] + static_cast<int64_t>(n0) * a.w_cpitch[g],
                       static_cast<uint32_t>(wrows * a.w_cpitch[g]), cb);
    }
  }
  float acc[2][4];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;
  auto part = [&](int c) -> bool {
    const bool landed = ptx::mbar_wait_cycles(&bar[c], 0, kDecWaitLimit);
    if (!__syncthreads_or(!landed)) return true;
    if (threadIdx.x == 0) {
      atomicExch(status, static_cast<int>(MXS_ERR_TIMEOUT));
      if (c == 0) ptx::mbar_wait_cycles(&bar[1], 0, kDecWaitLimit);
    }
    return false;
  };
  if (a.stage_w) {
    if (!part(0)) return;
    dec_segment<0, true>(a, smem, sp, n0, acc);
    dec_segment<1, true>(a, smem, sp, n0, acc);
    if (!part(1)) return;
    dec_segment<2, true>(a, smem, sp, n0, acc);
  } else {
    if (!part(0)) return;
    dec_segment<0, false>(a, smem, sp, n0, acc);
    dec_segment<1, false>(a, smem, sp, n0, acc);
    if (!part(1)) return;
    dec_segment<2, false>(a, smem, sp, n0, acc);
  }
  // the warps' partial sums, added in warp order
  __syncthreads();
  float(*red)[16][kDecRows + 1] = reinterpret_cast<float(*)[16][kDecRows + 1]>(smem);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    red[warp][gid][8 * j + 2 * tig] = acc[j][0];
    red[warp][gid][8 * j + 2 * tig + 1] = acc[j][1];
    red[warp][gid + 8][8 * j + 2 * tig] = acc[j][2];
    red[warp][gid + 8][8 * j + 2 * tig + 1] = acc[j][3];
  }
  __syncthreads();
  {
    const int m = threadIdx.x >> 4, r = threadIdx.x & 15, n = n0 + r;
    if (m < a.M && n < a.N) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) sum += red[w][m][r];
      a.Y[static_cast<int64_t>(m) * a.ldy + n] = __float2bfloat16_rn(sum);
    }
  }
}

static int64_t small_smem_bytes(const SmallArgs &a) {
  const int64_t red = static_cast<int64_t>(kDecWarps) * 16 * (kDecRows + 1) * 4;
  return std::max<int64_t>(dec_smem_plan(a).bytes, red);
}

constexpr int64_t kDecSmemCap = 200 * 1024;

static SmallArgs small_args(const mxs_mxtensor *A, const mxs_mxtensor *W, void *Y, int64_t ldy) {
  SmallArgs a{};
  a.M = static_cast<int32_t>(A->rows);
  a.N = static_cast<int32_t>(W->rows);
  a.nb_total = 0;
  for (int g = 0; g < 3; ++g) {
    a.nb[g] = static_cast<int32_t>(A->lay.seg[g].k_pad / kBlock);
    a.nb_total += a.nb[g];
    a.a_codes[g] = A->codes[g];
    a.a_cpitch[g] = A->code_pitch[g];
    a.a_scales[g] = A->scales[g];
    a.a_spitch[g] = A->scale_pitch[g];
    a.w_codes[g] = W->codes[g];
    a.w_cpitch[g] = W->code_pitch[g];
    a.w_scales[g] = W->scales[g];
    a.w_spitch[g] = W->scale_pitch[g];
  }
  a.Y = reinterpret_cast<__nv_bfloat16 *>(Y);
  a.ldy = ldy;
  a.stage_w = 1;
  if (small_smem_bytes(a) > kDecSmemCap) a.stage_w = 0;   // W codes stream from global memory instead
  return a;
}

// True when the decode path takes this call (up to 16 activation rows whose
// packed rows fit in shared memory).
bool small_fits(const mxs_mxtensor *A, const mxs_mxtensor *W) {
  if (A->rows > kDecMaxM) return false;
  return small_smem_bytes(small_args(A, W, nullptr, 0)) <= kDecSmemCap;
}

// ------------------------------------------------------------- GEMV (M <= 4)
//
// With one to four activation rows the tensor core's 16-row MMA mostly
// multiplies zeros, and each block's scaling dominates the instruction
// count.  Here one warp takes one W row; each lane takes every 32nd block
// of it, widens the block's codes to signed bytes (code * 2^(8-m), as
// above) and forms the block's integer dot product with each activation row
// by eight dp4a, exact in int32, then adds it times the exact scale
// 2^(ea-6) * 2^(ew-6) to an fp32 sum; the lanes' sums are added by a
// shuffle tree.  The activation rows are widened once per CTA into shared
// memory (int8 bytes and float scales).  The dp4a issue rate bounds this
// path at larger M, which is why it stops at four rows.
constexpr int kGvMaxM = 4;
constexpr int kGvThreads = 128;
constexpr int kGvU = 2;                       // blocks per lane with W loads in flight together

__host__ __device__ inline int64_t gemv_smem_bytes(int M, int nb_total) {
  return static_cast<int64_t>(M) * nb_total * (kBlock + 4);
}

// The 8 words of one block widened to signed bytes from its raw packed words.
template <int G>
__device__ __forceinline__ void widen_block(const uint32_t (&w)[8], uint32_t (&o)[8]) {
  if constexpr (G == 2) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      o[2 * j] = widen4(w[j] & 0xFFFFu);
      o[2 * j + 1] = widen4(w[j] >> 16);
    }
  } else if constexpr (G == 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int pos = 24 * i, word = pos >> 5, off = pos & 31;
      uint32_t v = w[word] >> off;
      if (off > 8) v |= w[word + 1] << (32 - off);
      o[i] = widen6(v);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = w[i];
  }
}

__global__ void __launch_bounds__(kGvThreads) gemm_gemv_kernel(SmallArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int NB = a.nb_total, M = a.M;
  uint8_t *aq = smem;                                                  // [M][NB][32] widened codes
  float *as = reinterpret_cast<float *>(smem + static_cast<int64_t>(M) * NB * kBlock);   // [M][NB] scales
  // activations: one thread per (row, block)
  for (int i = threadIdx.x; i < M * NB; i += kGvThreads) {
    const int m = i / NB, gb = i - m * NB;
    int g, bb;
    small_locate(a, gb, g, bb);
    const int mb = seg_bits(g);
    const uint8_t *c = a.a_codes[g] + m * a.a_cpitch[g] + static_cast<int64_t>(bb) * kBlock * mb / 8;
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    for (int j = 0; j < mb; ++j) w[j] = *reinterpret_cast<const uint32_t *>(c + 4 * j);
    uint32_t o[8];
    if (g == 0) widen_block<0>(w, o);
    else if (g == 1) widen_block<1>(w, o);
    else widen_block<2>(w, o);
    uint4 *dst = reinterpret_cast<uint4 *>(aq + static_cast<int64_t>(i) * kBlock);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    as[i] = pow2f(static_cast<int>(a.a_scales[g][m * a.a_spitch[g] + bb]) - 127 - 6);
  }
  __syncthreads();
  const int nwarps = gridDim.x * (kGvThreads / 32);
  for (int n = blockIdx.x * (kGvThreads / 32) + warp; n < a.N; n += nwarps) {
    float acc[kGvMaxM] = {0.f, 0.f, 0.f, 0.f};
    for (int b0 = lane; b0 < NB; b0 += 32 * kGvU) {
      uint32_t raw[kGvU][8];
      uint8_t sw[kGvU];
      int gs[kGvU];
#pragma unroll
      for (int u = 0; u < kGvU; ++u) {
        const int gb = b0 + 32 * u;
        gs[u] = -1;
        if (gb < NB) {
          int g, bb;
          small_locate(a, gb, g, bb);
          gs[u] = g;
          const uint8_t *c = a.w_codes[g] + static_cast<int64_t>(n) * a.w_cpitch[g] + static_cast<int64_t>(bb) * kBlock * seg_bits(g) / 8;
          if (g == 2) {
            const uint4 x = __ldg(reinterpret_cast<const uint4 *>(c));
            raw[u][0] = x.x; raw[u][1] = x.y; raw[u][2] = x.z; raw[u][3] = x.w;
          } else if (g == 1) {
#pragma unroll
            for (int j = 0; j < 3; ++j) {
              const uint2 x = __ldg(reinterpret_cast<const uint2 *>(c) + j);
              raw[u][2 * j] = x.x;
              raw[u][2 * j + 1] = x.y;
            }
          } else {
            const uint4 x0 = __ldg(reinterpret_cast<const uint4 *>(c)), x1 = __ldg(reinterpret_cast<const uint4 *>(c) + 1);
            raw[u][0] = x0.x; raw[u][1] = x0.y; raw[u][2] = x0.z; raw[u][3] = x0.w;
            raw[u][4] = x1.x; raw[u][5] = x1.y; raw[u][6] = x1.z; raw[u][7] = x1.w;
          }
          sw[u] = __ldg(a.w_scales[g] + static_cast<int64_t>(n) * a.w_spitch[g] + bb);
        }
      }
#pragma unroll
      for (int u = 0; u < kGvU; ++u) {
        if (gs[u] < 0) continue;
        const int gb = b0 + 32 * u;
        uint32_t wq[8];
        if (gs[u] == 0) widen_block<0>(raw[u], wq);
        else if (gs[u] == 1) widen_block<1>(raw[u], wq);
        else widen_block<2>(raw[u], wq);
        const float fw = pow2f(static_cast<int>(sw[u]) - 127 - 6);
#pragma unroll
        for (int m = 0; m < kGvMaxM; ++m) {
          if (m >= M) break;
          const uint4 *ap = reinterpret_cast<const uint4 *>(aq + (static_cast<int64_t>(m) * NB + gb) * kBlock);
          const uint4 x0 = ap[0], x1 = ap[1];
          int d = __dp4a(static_cast<int>(wq[0]), static_cast<int>(x0.x), 0);
          d = __dp4a(static_cast<int>(wq[1]), static_cast<int>(x0.y), d);
          d = __dp4a(static_cast<int>(wq[2]), static_cast<int>(x0.z), d);
          d = __dp4a(static_cast<int>(wq[3]), static_cast<int>(x0.w), d);
          d = __dp4a(static_cast<int>(wq[4]), static_cast<int>(x1.x), d);
          d = __dp4a(static_cast<int>(wq[5]), static_cast<int>(x1.y), d);
          d = __dp4a(static_cast<int>(wq[6]), static_cast<int>(x1.z), d);
          d = __dp4a(static_cast<int>(wq[7]), static_cast<int>(x1.w), d);
          acc[m] = fmaf(code_to_float(d), fw * as[m * NB + gb], acc[m]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < kGvMaxM; ++m) {
      if (m >= M) break;
      float v = acc[m];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) a.Y[static_cast<int64_t>(m) * a.ldy + n] = __float2bfloat16_rn(v);
    }
  }
}

mxs_status gemm_small(const mxs_mxtensor *A, const mxs_mxtensor *W, void *Y, int64_t ldy, cudaStream_t cs) {
  const SmallArgs a = small_args(A, W, Y, ldy);
  if (a.M <= kGvMaxM) {
    const int64_t gsmem = gemv_smem_bytes(a.M, a.nb_total);
    if (gsmem <= kDecSmemCap) {
      int dev = 0, nsm = 148;
      cudaGetDevice(&dev);
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
      if (!ensure_smem(gemm_gemv_kernel, static_cast<int>(std::max<int64_t>(gsmem, 16)))) return MXS_ERR_CUDA;
      // one resident wave: every CTA widens the activations once, then its
      // warps take W rows until none are left
      int occ = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gemm_gemv_kernel, kGvThreads,
                                                        static_cast<size_t>(std::max<int64_t>(gsmem, 16))) != cudaSuccess ||
          occ < 1)
        occ = 1;
      const int rows_per_cta = kGvThreads / 32;
      const int grid = static_cast<int>(std::min<int64_t>((a.N + rows_per_cta - 1) / rows_per_cta,
                                                          static_cast<int64_t>(nsm) * occ));
      launch_pdl(gemm_gemv_kernel, dim3(grid), dim3(kGvThreads), static_cast<size_t>(std::max<int64_t>(gsmem, 16)), cs, a);
      count_launch();
      return cuda_status(cudaGetLastError());
    }
  }
  int *status = device_status_word();
  if (!status) return MXS_ERR_CUDA;
  const int smem = static_cast<int>(small_smem_bytes(a));
  if (!ensure_smem(gemm_small_kernel, smem)) return MXS_ERR_CUDA;
  launch_pdl(gemm_small_kernel, dim3((a.N + kDecRows - 1) / kDecRows), dim3(kDecThreads), smem, cs, a, status);
  count_launch();
  return cuda_status(cudaGetLastError());
}


}  // namespace mxs
