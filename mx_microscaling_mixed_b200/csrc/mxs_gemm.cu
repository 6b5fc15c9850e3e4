// mxs_gemm.cu -- the mixed-width MXINT linear layer Y = deq(A) deq(W)^T on
// the B200 tensor cores (tcgen05, TMEM accumulators, TMA-fed shared memory).
//
// MXSens (arXiv 2607.17733), technical summary §2.3 last paragraph (the mixed
// mantissa widths ride on MXINT's block structure, no architecture change) and
// §4 (at a 4.03-bit budget ~1% of the work is wider than 4 bits, an estimated
// ~3% latency overhead).  The pages give no kernel; this design is for sm_100a.
//
// Exactness.  An m-bit MXINT value is q * 2^(e-m+2).
//   * 4-bit codes (|q| <= 7): q/4 is exact in FP8 E4M3 and the block's E8M0
//     byte is exactly the hardware block scale, so the 4-bit segment runs as
//     tcgen05 kind::mxf8f6f4 with 32-element block scaling: every product
//     q_a/4 * 2^ea * q_w/4 * 2^ew is the exact product of decoded values.
//   * 6/8-bit codes (|q| <= 127): not exact in any 8-bit float, but
//     q * 2^(e-m+2) has <= 7 significant bits and exponent >= -133, so it is
//     exact in bf16; these segments run as kind::f16 (bf16 x bf16).
// Both kinds accumulate into ONE fp32 accumulator in tensor memory; the
// epilogue rounds it once to bf16 (nearest even).
//
// Pipeline.  (1) A staging kernel re-codes both packed operands into the
// workspace: E4M3 bytes + E8M0 scales (in the tensor core's 512-byte scale
// chunk layout) for the 4-bit segment, bf16 values for the 8- and 6-bit
// segments.  (2) The GEMM kernel: one CTA per 128 x BN output tile; warp 0
// issues TMA loads (128-byte swizzled K-major tiles, one 128-byte K slice per
// stage for either kind) and bulk copies of the scale chunks; warp 1 owns the
// tensor memory and issues the MMAs (4 per stage) from one thread, copying
// the stage's scale chunks into tensor memory with tcgen05.cp first; warps
// 2-5 drain the accumulator (tcgen05.ld) to bf16.  Every wait is bounded: on
// expiry the kernel records MXS_ERR_TIMEOUT in a device status word, stops
// issuing, releases its tensor memory and returns.
#include <cuda.h>
#include <cuda_fp8.h>

#include <algorithm>
#include <mutex>

#include "mxs_internal.cuh"

namespace mxs {

__device__ int g_gemm_status = 0;

namespace ptx {

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_mxf8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                         uint32_t sfa, uint32_t sfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}
__device__ __forceinline__ void copy_sf_to_tmem(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row groups
// 1024 bytes apart; the start address may move by 32-byte K steps inside the
// 128-byte swizzle atom (tiles are 1024-byte aligned).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}
// Descriptor of one 512-byte scale chunk for tcgen05.cp 32x128b: 32 rows of
// 16 bytes, no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(128 >> 4) << 32) |
         (static_cast<uint64_t>(1) << 46);
}

}  // namespace ptx

constexpr int kBM = 128;           // output rows per CTA (A rows)
constexpr int kBN = 256;           // output columns per CTA (W rows)
constexpr int kStages = 4;
constexpr int kSliceBytes = 128;   // bytes of K per row per stage (64 bf16 or 128 fp8)
constexpr int kABytes = kBM * kSliceBytes;
constexpr int kBBytes = kBN * kSliceBytes;
constexpr int kSfChunk = 512;      // 128 rows x 4 block scales
constexpr int kSfaBytes = kSfChunk;
constexpr int kSfbBytes = (kBN / 128) * kSfChunk;
constexpr int kTmemCols = 512;
constexpr int kSfaCol = kBN;       // tensor-memory columns of the scale copies
constexpr int kSfbCol = kBN + 4;
constexpr int kGemmThreads = 192;
constexpr long long kWaitLimit = 4000000000LL;   // cycles (~2 s): then give up

// kind::f16: D fp32 (bits 4-5 = 1), A bf16 (bits 7-9 = 1), B bf16 (bits
// 10-12 = 1), both K-major, N>>3 at bit 17, M>>4 at bit 24.
constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) |
                                (static_cast<uint32_t>(kBN >> 3) << 17) | (static_cast<uint32_t>(kBM >> 4) << 24);
// kind::mxf8f6f4 block-scaled: A, B E4M3 (0), N>>3 at bit 17, E8M0 scales
// (bit 23), M>>4 at bit 24; the B/A scale byte ids go to bits 4-5 / 29-30.
constexpr uint32_t kIdescMxf8 = (static_cast<uint32_t>(kBN >> 3) << 17) | (1u << 23) |
                                (static_cast<uint32_t>(kBM >> 4) << 24);

struct GemmSmem {
  static constexpr int a_off = 0;
  static constexpr int b_off = a_off + kStages * kABytes;
  static constexpr int sfa_off = b_off + kStages * kBBytes;
  static constexpr int sfb_off = sfa_off + kStages * kSfaBytes;
  static constexpr int bar_off = sfb_off + kStages * kSfbBytes;
  static constexpr int bytes = bar_off + (2 * kStages + 1) * 8 + 16;
};
constexpr int kGemmSmemBytes = GemmSmem::bytes + 1024;   // + alignment slack

struct GemmArgs {
  int32_t M, N;
  int32_t n16_stages, n8_stages;
  int32_t nrg_a, nrg_b;            // 128-row groups in the scale chunk arrays
  const uint8_t *sfa, *sfb;
  __nv_bfloat16 *Y;
  int64_t ldy;
  int32_t y_vec;                   // 16-byte stores allowed
};

__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (;;) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimit) {
      *abort_flag = 1;
      atomicExch(&g_gemm_status, static_cast<int>(MXS_ERR_TIMEOUT));
      return false;
    }
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA16, const __grid_constant__ CUtensorMap tmB16,
                   const __grid_constant__ CUtensorMap tmA8, const __grid_constant__ CUtensorMap tmB8,
                   GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + GemmSmem::bar_off);
  uint64_t *empty = full + kStages;
  uint64_t *accum_full = empty + kStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum_full + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * kBM;
  const int n_iters = g.n16_stages + g.n8_stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accum_full, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % kStages;
        if (it >= kStages && !wait_bounded(&empty[s], ((it / kStages) - 1) & 1, abort_flag)) break;
        uint8_t *sa = smem + GemmSmem::a_off + s * kABytes;
        uint8_t *sb = smem + GemmSmem::b_off + s * kBBytes;
        if (it < g.n16_stages) {
          ptx::mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
          ptx::tma_load_2d(sa, &tmA16, &full[s], it * 64, m0);
          ptx::tma_load_2d(sb, &tmB16, &full[s], it * 64, n0);
        } else {
          const int j = it - g.n16_stages;
          ptx::mbar_arrive_expect_tx(&full[s], kABytes + kBBytes + kSfaBytes + kSfbBytes);
          ptx::tma_load_2d(sa, &tmA8, &full[s], j * 128, m0);
          ptx::tma_load_2d(sb, &tmB8, &full[s], j * 128, n0);
          ptx::bulk_load(smem + GemmSmem::sfa_off + s * kSfaBytes,
                         g.sfa + (static_cast<int64_t>(j) * g.nrg_a + m0 / 128) * kSfChunk, kSfaBytes, &full[s]);
          ptx::bulk_load(smem + GemmSmem::sfb_off + s * kSfbBytes,
                         g.sfb + (static_cast<int64_t>(j) * g.nrg_b + n0 / 128) * kSfChunk, kSfbBytes, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t tsfa = tmem + kSfaCol, tsfb = tmem + kSfbCol;
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % kStages;
        if (!wait_bounded(&full[s], (it / kStages) & 1, abort_flag)) break;
        ptx::tc_fence_after();
        const uint32_t a_base = ptx::smem_addr(smem + GemmSmem::a_off + s * kABytes);
        const uint32_t b_base = ptx::smem_addr(smem + GemmSmem::b_off + s * kBBytes);
        if (it < g.n16_stages) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_bf16(tmem, ptx::desc_sw128(a_base + 32 * k), ptx::desc_sw128(b_base + 32 * k), kIdescBf16,
                          (it > 0 || k > 0) ? 1u : 0u);
        } else {
          const uint32_t sfa_s = ptx::smem_addr(smem + GemmSmem::sfa_off + s * kSfaBytes);
          const uint32_t sfb_s = ptx::smem_addr(smem + GemmSmem::sfb_off + s * kSfbBytes);
          ptx::copy_sf_to_tmem(tsfa, ptx::desc_sf(sfa_s));
#pragma unroll
          for (int c = 0; c < kBN / 128; ++c) ptx::copy_sf_to_tmem(tsfb + 4 * c, ptx::desc_sf(sfb_s + kSfChunk * c));
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t idesc = kIdescMxf8 | (static_cast<uint32_t>(k) << 4) | (static_cast<uint32_t>(k) << 29);
            ptx::mma_mxf8(tmem, ptx::desc_sw128(a_base + 32 * k), ptx::desc_sw128(b_base + 32 * k), idesc,
                          (it > 0 || k > 0) ? 1u : 0u, tsfa | (static_cast<uint32_t>(k) << 30),
                          tsfb | (static_cast<uint32_t>(k) << 30));
          }
        }
        ptx::mma_commit(&empty[s]);
      }
      ptx::mma_commit(accum_full);
    }
  } else {
    // Epilogue: warp w may read tensor-memory lanes 32*(w%4) .. 32*(w%4)+31.
    const bool ok = wait_bounded(accum_full, 0, abort_flag);
    ptx::tc_fence_after();
    if (ok && !*abort_flag) {
      const int q = warp & 3;
      const int row = m0 + q * 32 + lane;
      __nv_bfloat16 *yrow = g.Y + static_cast<int64_t>(row) * g.ldy;
      for (int c = 0; c < kBN; c += 16) {
        uint32_t r[16];
        ptx::tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + c, r);
        ptx::tmem_wait_ld();
        if (row >= g.M) continue;
        const int n = n0 + c;
        if (g.y_vec && n + 16 <= g.N) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            pk[i] = *reinterpret_cast<uint32_t *>(&h);
          }
          uint4 *dst = reinterpret_cast<uint4 *>(yrow + n);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (n + i < g.N) yrow[n + i] = __float2bfloat16_rn(__uint_as_float(r[i]));
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- staging

struct StageOperand {
  int64_t rows;
  const uint8_t *codes[3];
  int64_t cpitch[3];
  const uint8_t *scales[3];
  int64_t spitch[3];
  __nv_bfloat16 *x16;   // rows x k16 (8-bit then 6-bit segment values)
  uint8_t *x8;          // rows x k4 E4M3 bytes
  uint8_t *sf;          // scale chunks [k-group][row-group][512]
  int32_t nrg;          // row groups of 128 in sf
};

struct StageArgs {
  StageOperand op[2];
  int32_t nb[3];        // blocks per segment
  int32_t nb_total;
  int64_t k16, k4;
  int64_t k6_off16;     // start of the 6-bit segment inside x16 rows
  int32_t nkg;          // k-groups of 4 blocks in the 4-bit segment
  int64_t n_decode[2];  // rows * nb_total per operand
  int64_t n_pad[2];     // scale-chunk entries per operand (all, incl. padding)
};

__device__ __forceinline__ int64_t sf_index(int64_t r, int64_t b, int32_t nrg) {
  return ((b >> 2) * nrg + (r >> 7)) * kSfChunk + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}

__device__ __forceinline__ int unpack_code(const uint8_t *c, int t, int m) {
  if (m == 8) return static_cast<int8_t>(c[t]);
  if (m == 4) {
    const int v = (c[t >> 1] >> (4 * (t & 1))) & 0xF;
    return v >= 8 ? v - 16 : v;
  }
  const int grp = t >> 2, sub = t & 3;
  const uint32_t w = c[3 * grp] | (c[3 * grp + 1] << 8) | (c[3 * grp + 2] << 16);
  const int v = (w >> (6 * sub)) & 0x3F;
  return v >= 32 ? v - 64 : v;
}

__global__ void __launch_bounds__(256) gemm_stage_kernel(StageArgs a) {
  const int64_t total = a.n_decode[0] + a.n_decode[1] + a.n_pad[0] + a.n_pad[1];
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int64_t w = i;
    if (w < a.n_decode[0] + a.n_decode[1]) {
      const int o = w < a.n_decode[0] ? 0 : 1;
      if (o) w -= a.n_decode[0];
      const StageOperand &op = a.op[o];
      const int64_t row = w / a.nb_total;
      int blk = static_cast<int>(w - row * a.nb_total);
      int g = 0;
      while (blk >= a.nb[g]) { blk -= a.nb[g]; ++g; }
      const int m = seg_bits(g);
      const uint8_t *c = op.codes[g] + row * op.cpitch[g] + static_cast<int64_t>(blk) * kBlock * m / 8;
      const uint8_t sbyte = op.scales[g][row * op.spitch[g] + blk];
      if (g == 2) {
        __align__(16) uint8_t out[kBlock];
#pragma unroll
        for (int t = 0; t < kBlock; t += 2) {
          const float2 f = make_float2(0.25f * static_cast<float>(unpack_code(c, t, 4)),
                                       0.25f * static_cast<float>(unpack_code(c, t + 1, 4)));
          const __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
          out[t] = static_cast<uint8_t>(p & 0xFF);
          out[t + 1] = static_cast<uint8_t>(p >> 8);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(op.x8 + row * a.k4 + static_cast<int64_t>(blk) * kBlock);
        dst[0] = *reinterpret_cast<uint4 *>(out);
        dst[1] = *reinterpret_cast<uint4 *>(out + 16);
        op.sf[sf_index(row, blk, op.nrg)] = sbyte;
      } else {
        const float step = pow2f(static_cast<int>(sbyte) - 127 - m + 2);
        __align__(16) __nv_bfloat16 out[kBlock];
#pragma unroll
        for (int t = 0; t < kBlock; ++t) out[t] = __float2bfloat16_rn(static_cast<float>(unpack_code(c, t, m)) * step);
        const int64_t col = (g == 0 ? 0 : a.k6_off16) + static_cast<int64_t>(blk) * kBlock;
        uint4 *dst = reinterpret_cast<uint4 *>(op.x16 + row * a.k16 + col);
        const uint4 *src = reinterpret_cast<const uint4 *>(out);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[v] = src[v];
      }
    } else {
      // neutral scale (2^0) for chunk entries outside the real rows / blocks
      w -= a.n_decode[0] + a.n_decode[1];
      const int o = w < a.n_pad[0] ? 0 : 1;
      if (o) w -= a.n_pad[0];
      const StageOperand &op = a.op[o];
      const int64_t nbp = static_cast<int64_t>(a.nkg) * 4;
      const int64_t row = w / nbp, blk = w - row * nbp;
      if (row >= op.rows || blk >= a.nb[2]) op.sf[sf_index(row, blk, op.nrg)] = 127;
    }
  }
}

// ---------------------------------------------------------------- host side

struct WsPlan {
  int64_t k16, k4;
  int32_t nkg, nrg_a, nrg_b;
  size_t off_a16, off_b16, off_a8, off_b8, off_sfa, off_sfb, total;
};

static WsPlan plan_workspace(const mxs_mxtensor *A, const mxs_mxtensor *W) {
  WsPlan p{};
  const int64_t M = A->rows, N = W->rows;
  p.k16 = A->lay.seg[0].k_pad + A->lay.seg[1].k_pad;
  p.k4 = A->lay.seg[2].k_pad;
  p.nkg = static_cast<int32_t>((p.k4 + 127) / 128);
  p.nrg_a = static_cast<int32_t>((M + kBM - 1) / kBM);
  p.nrg_b = static_cast<int32_t>((N + kBN - 1) / kBN * (kBN / 128));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += static_cast<size_t>(round_up(static_cast<int64_t>(bytes), 1024));
    return o;
  };
  p.off_a16 = take(static_cast<size_t>(M * p.k16 * 2));
  p.off_b16 = take(static_cast<size_t>(N * p.k16 * 2));
  p.off_a8 = take(static_cast<size_t>(M * p.k4));
  p.off_b8 = take(static_cast<size_t>(N * p.k4));
  p.off_sfa = take(static_cast<size_t>(p.nkg) * p.nrg_a * kSfChunk);
  p.off_sfb = take(static_cast<size_t>(p.nkg) * p.nrg_b * kSfChunk);
  p.total = off;
  return p;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
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

// 2-D K-major tile map: inner dimension K (elements), outer `rows`, box
// 128 bytes x box_rows, 128-byte swizzle, zero fill out of bounds.
static bool make_map(CUtensorMap *m, CUtensorMapDataType dt, int esize, void *base, int64_t k, int64_t rows,
                     int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(k * esize)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kSliceBytes / esize), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool same_layout(const mxs_layout &a, const mxs_layout &b) {
  if (a.K != b.K || a.K_pad != b.K_pad || a.perm != b.perm) return false;
  for (int g = 0; g < 3; ++g)
    if (a.seg[g].k_real != b.seg[g].k_real) return false;
  return true;
}

static mxs_status gemm_check(const mxs_mxtensor *A, const mxs_mxtensor *W) {
  if (!A || !W) return MXS_ERR_ARG;
  mxs_status st = check_mxtensor(A);
  if (st != MXS_OK) return st;
  if ((st = check_mxtensor(W)) != MXS_OK) return st;
  if (!same_layout(A->lay, W->lay)) return MXS_ERR_SHAPE;
  if (A->rows > INT32_MAX / 2 || W->rows > INT32_MAX / 2) return MXS_ERR_SHAPE;
  return MXS_OK;
}

}  // namespace mxs

using namespace mxs;

extern "C" mxs_status mxs_sync(void *stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MXS_ERR_CUDA;
  int st = 0;
  if (cudaMemcpyFromSymbol(&st, g_gemm_status, sizeof(int)) != cudaSuccess) return MXS_ERR_CUDA;
  if (st != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_gemm_status, &zero, sizeof(int));
    return static_cast<mxs_status>(st);
  }
  return MXS_OK;
}

extern "C" mxs_status mxs_gemm_workspace_bytes(const mxs_mxtensor *A, const mxs_mxtensor *W, size_t *bytes) {
  if (!bytes) return MXS_ERR_ARG;
  mxs_status st = gemm_check(A, W);
  if (st != MXS_OK) return st;
  *bytes = plan_workspace(A, W).total;
  return MXS_OK;
}

extern "C" mxs_status mxs_gemm(const mxs_mxtensor *A, const mxs_mxtensor *W, void *Y, int64_t ldy, void *ws,
                               size_t ws_bytes, void *stream) {
  mxs_status st = gemm_check(A, W);
  if (st != MXS_OK) return st;
  const int64_t M = A->rows, N = W->rows;
  if (ldy < N) return MXS_ERR_SHAPE;
  if (M == 0 || N == 0) return MXS_OK;
  if (!Y) return MXS_ERR_ARG;
  if ((st = check_device()) != MXS_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (A->lay.K_pad == 0) {
    count_launch();
    return cuda_status(cudaMemset2DAsync(Y, static_cast<size_t>(ldy) * 2, 0, static_cast<size_t>(N) * 2,
                                         static_cast<size_t>(M), cs));
  }
  const WsPlan p = plan_workspace(A, W);
  if (!ws || ws_bytes < p.total || (reinterpret_cast<uintptr_t>(ws) & 1023u)) return MXS_ERR_WORKSPACE;
  uint8_t *base = reinterpret_cast<uint8_t *>(ws);

  StageArgs sa{};
  const mxs_mxtensor *ops[2] = {A, W};
  for (int o = 0; o < 2; ++o) {
    StageOperand &op = sa.op[o];
    op.rows = ops[o]->rows;
    for (int g = 0; g < 3; ++g) {
      op.codes[g] = ops[o]->codes[g];
      op.cpitch[g] = ops[o]->code_pitch[g];
      op.scales[g] = ops[o]->scales[g];
      op.spitch[g] = ops[o]->scale_pitch[g];
    }
    op.x16 = reinterpret_cast<__nv_bfloat16 *>(base + (o ? p.off_b16 : p.off_a16));
    op.x8 = base + (o ? p.off_b8 : p.off_a8);
    op.sf = base + (o ? p.off_sfb : p.off_sfa);
    op.nrg = o ? p.nrg_b : p.nrg_a;
  }
  sa.nb_total = 0;
  for (int g = 0; g < 3; ++g) {
    sa.nb[g] = static_cast<int32_t>(A->lay.seg[g].k_pad / kBlock);
    sa.nb_total += sa.nb[g];
  }
  sa.k16 = p.k16;
  sa.k4 = p.k4;
  sa.k6_off16 = A->lay.seg[0].k_pad;
  sa.nkg = p.nkg;
  sa.n_decode[0] = M * sa.nb_total;
  sa.n_decode[1] = N * sa.nb_total;
  sa.n_pad[0] = static_cast<int64_t>(p.nrg_a) * 128 * p.nkg * 4;
  sa.n_pad[1] = static_cast<int64_t>(p.nrg_b) * 128 * p.nkg * 4;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t total = sa.n_decode[0] + sa.n_decode[1] + sa.n_pad[0] + sa.n_pad[1];
  const int sgrid = static_cast<int>(std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(nsm) * 16));
  gemm_stage_kernel<<<sgrid, 256, 0, cs>>>(sa);
  count_launch();

  CUtensorMap mA16{}, mB16{}, mA8{}, mB8{};
  if (p.k16 > 0) {
    if (!make_map(&mA16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base + p.off_a16, p.k16, M, kBM) ||
        !make_map(&mB16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base + p.off_b16, p.k16, N, kBN))
      return MXS_ERR_CUDA;
  }
  if (p.k4 > 0) {
    if (!make_map(&mA8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base + p.off_a8, p.k4, M, kBM) ||
        !make_map(&mB8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base + p.off_b8, p.k4, N, kBN))
      return MXS_ERR_CUDA;
  }
  GemmArgs ga{};
  ga.M = static_cast<int32_t>(M);
  ga.N = static_cast<int32_t>(N);
  ga.n16_stages = static_cast<int32_t>((p.k16 + 63) / 64);
  ga.n8_stages = static_cast<int32_t>((p.k4 + 127) / 128);
  ga.nrg_a = p.nrg_a;
  ga.nrg_b = p.nrg_b;
  ga.sfa = base + p.off_sfa;
  ga.sfb = base + p.off_sfb;
  ga.Y = reinterpret_cast<__nv_bfloat16 *>(Y);
  ga.ldy = ldy;
  ga.y_vec = aligned16(Y) && (ldy * 2) % 16 == 0;
  static bool attr_set[64] = {};
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) !=
        cudaSuccess)
      return MXS_ERR_CUDA;
    attr_set[dev] = true;
  }
  dim3 grid(static_cast<unsigned>((N + kBN - 1) / kBN), static_cast<unsigned>((M + kBM - 1) / kBM));
  gemm_tc_kernel<<<grid, kGemmThreads, kGemmSmemBytes, cs>>>(mA16, mB16, mA8, mB8, ga);
  count_launch();
  return cuda_status(cudaGetLastError());
}
