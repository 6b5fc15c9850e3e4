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
#include "mxs_ptx.cuh"
#include "mxs_decode.cuh"

namespace mxs {

__device__ int g_status = 0;

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
// The scale copies rotate through kSfSlots slots of kSfSlotCols columns, so a
// stage's copies never overwrite the scales the previous stage's MMAs still
// read: the copy does not wait for those MMAs (256 + 4 x 12 = 304 of 512
// columns).
constexpr int kSfSlots = 4;
constexpr int kSfSlotCols = 12;
constexpr int kGemmThreads = 192;
constexpr long long kWaitLimit = 4000000000LL;   // cycles (~2 s): then give up
// Limit of the pipeline waits of the two tensor-core kernels (mxs_set_wait_limit
// lowers it for a diagnostic run).  The drains on the way out keep kWaitLimit.
__device__ long long g_wait_limit = kWaitLimit;

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
  // full[S], empty[S], accum_full, drain; tmem slot, abort flag
  static constexpr int bytes = bar_off + (2 * kStages + 2) * 8 + 16;
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
  const long long t0 = clock64(), limit = g_wait_limit;
  for (;;) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      atomicExch(&g_status, static_cast<int>(MXS_ERR_TIMEOUT));
      return false;
    }
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA16, const __grid_constant__ CUtensorMap tmB16,
                   const __grid_constant__ CUtensorMap tmA8, const __grid_constant__ CUtensorMap tmB8,
                   GemmArgs g) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + GemmSmem::bar_off);
  uint64_t *empty = full + kStages;
  uint64_t *accum_full = empty + kStages;
  uint64_t *drain = accum_full + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
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
    ptx::mbar_init(drain, 1);
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
  int issued = 0;                                    // stages whose copies the producer issued

  if (warp == 0) {
    if (lane == 0) {
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % kStages;
        if (it >= kStages && !wait_bounded(&empty[s], ((it / kStages) - 1) & 1, abort_flag)) break;
        issued = it + 1;
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
          const uint32_t slot = kSfSlotCols * static_cast<uint32_t>(it % kSfSlots);
          ptx::copy_sf_to_tmem(tsfa + slot, ptx::desc_sf(sfa_s));
#pragma unroll
          for (int c = 0; c < kBN / 128; ++c)
            ptx::copy_sf_to_tmem(tsfb + slot + 4 * c, ptx::desc_sf(sfb_s + kSfChunk * c));
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t idesc = kIdescMxf8 | (static_cast<uint32_t>(k) << 4) | (static_cast<uint32_t>(k) << 29);
            ptx::mma_mxf8(tmem, ptx::desc_sw128(a_base + 32 * k), ptx::desc_sw128(b_base + 32 * k), idesc,
                          (it > 0 || k > 0) ? 1u : 0u, (tsfa + slot) | (static_cast<uint32_t>(k) << 30),
                          (tsfb + slot) | (static_cast<uint32_t>(k) << 30));
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
  if (*abort_flag) {
    // Given up: the copies already issued land and the MMAs already issued
    // finish before the CTA frees its tensor memory and leaves (each wait
    // bounded by the full limit).
    if (warp == 0 && lane == 0)
      for (int i = max(0, issued - kStages); i < issued; ++i)
        ptx::mbar_wait_cycles(&full[i % kStages], (i / kStages) & 1, kWaitLimit);
    if (warp == 1 && lane == 0) {
      ptx::mma_commit(drain);
      ptx::mbar_wait_cycles(drain, 0, kWaitLimit);
    }
    ptx::tc_fence_before();
    __syncthreads();
  }
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------- 2-CTA persistent kernel
//
// A cluster of two CTAs computes 256 x 256 output tiles with cta_group::2
// MMAs: each CTA stages its own 128 rows of A and its own 128 rows (half of
// N) of B, the leader issues M=256, N=256 MMAs that read both CTAs' shared
// memory and write each CTA's 128-row half of the accumulator into that
// CTA's tensor memory.  Per pair this halves the B tile traffic of the
// 1-CTA kernel.  Both CTAs' TMA copies complete on the leader's "full"
// barriers; the MMA commits arrive on both CTAs' "empty" barriers.  The
// 4-bit segment's scales: each CTA holds its own 128 A-row chunk and the
// full 256 N-row pair of chunks (the MMA needs all N scales in each CTA).
// CTAs are persistent: pair p takes tiles p, p + pairs, ...; eight epilogue
// warps per CTA drain the accumulator into registers, release it to the
// leader (one arrival per warp per CTA) and store bf16 while the next tile's
// MMAs already run.

namespace ptx {
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}
// lowers the barrier's pending transaction count by `bytes` without a copy
__device__ __forceinline__ void mbar_complete_tx(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t leader_bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t *slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma2_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma2_mxf8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                          uint32_t sfa, uint32_t sfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}
__device__ __forceinline__ void mma2_commit_both(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void copy_sf_to_tmem2(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
}  // namespace ptx

constexpr int kP2Stages = 3;
constexpr int kP2Sub = 2;                          // K slices per stage: 8 MMAs per barrier round
constexpr int kP2Rows = 128;                       // rows of A per CTA per stage
constexpr int kP2N = 240;                          // output columns per pair tile (W rows)
constexpr int kP2BRows = kP2N / 2;                 // rows of B per CTA per stage
constexpr int kP2AccCols = kP2N;                   // one accumulator buffer; two buffers at columns 0 and 240
constexpr int kP2SfCol = 2 * kP2AccCols;           // scale slots from column 480: 2 x 12 columns
constexpr int kP2SfSlots = 2;                      // scale slots, taken by slices in turn
static_assert(kP2SfCol + kP2SfSlots * kSfSlotCols <= kTmemCols, "accumulators and scale slots fit in TMEM");
constexpr int kP2TileBytes = kP2Rows * kSliceBytes;
constexpr int kP2SfaBytes = kSfChunk;              // own 128 A rows x 4 blocks
constexpr int kP2SfbBytes = 2 * kSfChunk;          // the pair's 256 N rows x 4 blocks
constexpr int kP2EpiWarps = 8;
constexpr int kP2EpiCols = 40;                      // Y columns per TMA store (3 per half tile)
constexpr int kP2Threads = (2 + kP2EpiWarps) * 32;
// cta_group::2, M = 256, N = 240
constexpr uint32_t kIdesc2Bf16 = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kP2N >> 3) << 17) |
                                 (static_cast<uint32_t>(256 >> 4) << 24);
constexpr uint32_t kIdesc2Mxf8 = (static_cast<uint32_t>(kP2N >> 3) << 17) | (1u << 23) |
                                 (static_cast<uint32_t>(256 >> 4) << 24);

struct P2Smem {
  static constexpr int a_off = 0;
  static constexpr int b_off = a_off + kP2Stages * kP2Sub * kP2TileBytes;
  static constexpr int sfa_off = b_off + kP2Stages * kP2Sub * kP2TileBytes;
  static constexpr int sfb_off = sfa_off + kP2Stages * kP2Sub * kP2SfaBytes;
  static constexpr int bar_off = sfb_off + kP2Stages * kP2Sub * kP2SfbBytes;
  // full[S], empty[S], acc_full[2], acc_empty[2], drain; tmem slot, abort
  // flag, issued-stage count
  static constexpr int bar_end = bar_off + (2 * kP2Stages + 5) * 8 + 16;
  // per epilogue warp: a 32-row x 40-column bf16 piece of Y on its way out by TMA
  static constexpr int epi_off = (bar_end + 127) / 128 * 128;
  static constexpr int epi_bytes = 32 * kP2EpiCols * 2;
  static constexpr int bytes = epi_off + kP2EpiWarps * epi_bytes;
};
constexpr int kP2SmemBytes = P2Smem::bytes + 1024;

// Output tile t -> (mt, nt).  Tiles run through a group of kP2Raster
// m-tiles for one n-tile before moving to the next n-tile, so the ~74 tiles
// in flight at a time (one per pair) share about 8 m-tiles of A and 10
// n-tiles of W, which stay in L2 while the group is worked on: A is read
// from DRAM about once, W once per group.
constexpr int kP2Raster = 8;
__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles, int &mt, int &nt) {
  const int grp = t / (kP2Raster * n_tiles);
  const int rem = t - grp * (kP2Raster * n_tiles);
  const int gm = min(kP2Raster, m_tiles - grp * kP2Raster);     // m-tiles of this group
  nt = rem / gm;
  mt = grp * kP2Raster + (rem - nt * gm);
}

struct P2Args {
  int32_t M, N;
  int32_t n16_stages, n8_stages;
  int32_t m_tiles, n_tiles;
  int32_t nrg_a, nrg_b;
  __nv_bfloat16 *Y;
  int64_t ldy;
  int32_t y_vec;
  int32_t y_tma;         // Y leaves through the tensor map (16-byte aligned rows)
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kP2Threads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA16, const __grid_constant__ CUtensorMap tmB16,
                    const __grid_constant__ CUtensorMap tmA8, const __grid_constant__ CUtensorMap tmB8,
                    const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                    const __grid_constant__ CUtensorMap tmY, P2Args g) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + P2Smem::bar_off);
  uint64_t *empty = full + kP2Stages;
  uint64_t *acc_full = empty + kP2Stages;             // [2]: one per accumulator buffer
  uint64_t *acc_empty = acc_full + 2;                 // [2]
  uint64_t *drain = acc_empty + 2;                    // the MMAs issued have finished
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *issued_slot = reinterpret_cast<int *>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int n16s = (g.n16_stages + kP2Sub - 1) / kP2Sub, n8s = (g.n8_stages + kP2Sub - 1) / kP2Sub;
  const int n_iters = n16s + n8s;                      // stages of kP2Sub slices
  const int n_tiles_total = g.m_tiles * g.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kP2Stages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&acc_full[b], 1);
      ptx::mbar_init(&acc_empty[b], 2 * kP2EpiWarps);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc2(tmem_slot, kTmemCols);
    ptx::tmem_relinquish2();
  }
  if (threadIdx.x == 32) {
    const CUtensorMap *maps[7] = {&tmA16, &tmB16, &tmA8, &tmB8, &tmSFA, &tmSFB, &tmY};
    for (int i = 0; i < 7; ++i) asm volatile("prefetch.tensormap [%0];" ::"l"(maps[i]) : "memory");
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the staged operands and Y belong to earlier kernels in the stream
  pdl_wait();
  // bytes of one K slice, both CTAs
  constexpr uint32_t bytes16 = 2 * (kP2TileBytes + kP2BRows * kSliceBytes);
  constexpr uint32_t bytes8 = 2 * (kP2TileBytes + kP2BRows * kSliceBytes + kP2SfaBytes + kP2SfbBytes);
  int it = 0;                                         // producer: stages whose copies were issued

  if (warp == 0) {
    if (lane == 0) {
      for (int t = pair; t < n_tiles_total && !*abort_flag; t += npairs) {
        int mt, nt;
        tile_coords(t, g.m_tiles, g.n_tiles, mt, nt);
        const int am = mt * 256 + static_cast<int>(rank) * kP2Rows;      // this CTA's A rows
        const int bn = nt * kP2N + static_cast<int>(rank) * kP2BRows;    // this CTA's B rows
        for (int k = 0; k < n_iters; ++k, ++it) {
          const int s = it % kP2Stages;
          if (it >= kP2Stages && !wait_bounded(&empty[s], ((it / kP2Stages) - 1) & 1, abort_flag)) break;
          const uint32_t lbar = ptx::map_to_rank(ptx::smem_addr(&full[s]), 0);
          const bool wide = k < n16s;
          const int j0 = kP2Sub * (wide ? k : k - n16s);                    // first slice of the stage
          const int nsub = min(kP2Sub, (wide ? g.n16_stages : g.n8_stages) - j0);
          if (leader) ptx::mbar_arrive_expect_tx(&full[s], nsub * (wide ? bytes16 : bytes8));
          for (int h = 0; h < nsub; ++h) {
            const int j = j0 + h;
            uint8_t *sa = smem + P2Smem::a_off + (s * kP2Sub + h) * kP2TileBytes;
            uint8_t *sb = smem + P2Smem::b_off + (s * kP2Sub + h) * kP2TileBytes;
            if (wide) {
              ptx::tma_load_2d_pair(sa, &tmA16, lbar, j * 64, am);
              ptx::tma_load_2d_pair(sb, &tmB16, lbar, j * 64, bn);
            } else {
              ptx::tma_load_2d_pair(sa, &tmA8, lbar, j * 128, am);
              ptx::tma_load_2d_pair(sb, &tmB8, lbar, j * 128, bn);
              ptx::tma_load_2d_pair(smem + P2Smem::sfa_off + (s * kP2Sub + h) * kP2SfaBytes, &tmSFA, lbar, 0,
                                    4 * (j * g.nrg_a + am / 128));
              ptx::tma_load_2d_pair(smem + P2Smem::sfb_off + (s * kP2Sub + h) * kP2SfbBytes, &tmSFB, lbar, 0,
                                    4 * (j * g.nrg_b + nt * 2));
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      const uint32_t tsfa = tmem + kP2SfCol, tsfb = tsfa + 4;
      int it = 0, tl = 0;
      for (int t = pair; t < n_tiles_total && !*abort_flag; t += npairs, ++tl) {
        const int buf = tl & 1;
        const uint32_t acc = tmem + buf * kP2AccCols;
        // the buffer's previous tile (tl - 2) must have been drained
        if (tl >= 2 && !wait_bounded(&acc_empty[buf], ((tl >> 1) - 1) & 1, abort_flag)) break;
        ptx::tc_fence_after();
        bool ok = true;
        for (int k = 0; k < n_iters; ++k, ++it) {
          const int s = it % kP2Stages;
          if (!wait_bounded(&full[s], (it / kP2Stages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const bool wide = k < n16s;
          const int j0 = kP2Sub * (wide ? k : k - n16s);
          const int nsub = min(kP2Sub, (wide ? g.n16_stages : g.n8_stages) - j0);
          if (!wide) {
            // the stage's scale chunks first (slices take the slots in
            // turn), so the copies for a later slice are queued ahead of
            // the earlier slice's MMAs; a slot is reused only by a later
            // slice, behind these MMAs in the same issue order
            for (int h = 0; h < nsub; ++h) {
              const uint32_t sfa_s = ptx::smem_addr(smem + P2Smem::sfa_off + (s * kP2Sub + h) * kP2SfaBytes);
              const uint32_t sfb_s = ptx::smem_addr(smem + P2Smem::sfb_off + (s * kP2Sub + h) * kP2SfbBytes);
              const uint32_t slot = kSfSlotCols * static_cast<uint32_t>((it * kP2Sub + h) % kP2SfSlots);
              ptx::copy_sf_to_tmem2(tsfa + slot, ptx::desc_sf(sfa_s));
              ptx::copy_sf_to_tmem2(tsfb + slot, ptx::desc_sf(sfb_s));
              ptx::copy_sf_to_tmem2(tsfb + slot + 4, ptx::desc_sf(sfb_s + kSfChunk));
            }
          }
          for (int h = 0; h < nsub; ++h) {
            const uint32_t a_base = ptx::smem_addr(smem + P2Smem::a_off + (s * kP2Sub + h) * kP2TileBytes);
            const uint32_t b_base = ptx::smem_addr(smem + P2Smem::b_off + (s * kP2Sub + h) * kP2TileBytes);
            if (wide) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                ptx::mma2_bf16(acc, ptx::desc_sw128(a_base + 32 * q), ptx::desc_sw128(b_base + 32 * q), kIdesc2Bf16,
                               (k > 0 || h > 0 || q > 0) ? 1u : 0u);
            } else {
              const uint32_t slot = kSfSlotCols * static_cast<uint32_t>((it * kP2Sub + h) % kP2SfSlots);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint32_t idesc = kIdesc2Mxf8 | (static_cast<uint32_t>(q) << 4) | (static_cast<uint32_t>(q) << 29);
                ptx::mma2_mxf8(acc, ptx::desc_sw128(a_base + 32 * q), ptx::desc_sw128(b_base + 32 * q), idesc,
                               (k > 0 || h > 0 || q > 0) ? 1u : 0u, (tsfa + slot) | (static_cast<uint32_t>(q) << 30),
                               (tsfb + slot) | (static_cast<uint32_t>(q) << 30));
              }
            }
          }
          ptx::mma2_commit_both(&empty[s]);
        }
        if (!ok) break;
        ptx::mma2_commit_both(&acc_full[buf]);
      }
    }
  } else {
    // epilogue: warp w reads lanes 32*(w%4)..+31 and columns 120h..120h+119
    // (h = 0, 1) of the tile's accumulator buffer; loads are 32 columns wide,
    // so the last one reads 8 columns past the half, which are not stored
    const int q = warp & 3, h = (warp - 2) >> 2;
    int tl = 0;
    for (int t = pair; t < n_tiles_total; t += npairs, ++tl) {
      const int buf = tl & 1;
      if (!wait_bounded(&acc_full[buf], (tl >> 1) & 1, abort_flag)) break;
      ptx::tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        ptx::tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * kP2AccCols + (kP2N / 2) * h + 32 * c, r[c]);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&acc_empty[buf]), 0));
      int mt, nt;
      tile_coords(t, g.m_tiles, g.n_tiles, mt, nt);
      const int row0 = mt * 256 + static_cast<int>(rank) * kP2Rows + q * 32;
      if (g.y_tma) {
        // three 32 x 40 pieces per warp: bf16 rows into the warp's staging
        // buffer (row = lane, 80 bytes), then one tensor store each; the
        // store clips rows past M and columns past N
        uint8_t *stg = smem + P2Smem::epi_off + (warp - 2) * P2Smem::epi_bytes;
#pragma unroll
        for (int pc = 0; pc < kP2N / 2 / kP2EpiCols; ++pc) {
          uint32_t pk[kP2EpiCols / 2];
#pragma unroll
          for (int i = 0; i < kP2EpiCols / 2; ++i) {
            const int col = kP2EpiCols * pc + 2 * i;
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[col >> 5][col & 31]),
                                                      __uint_as_float(r[col >> 5][(col & 31) + 1]));
            pk[i] = *reinterpret_cast<uint32_t *>(&b2);
          }
          if (lane == 0) ptx::bulk_wait_read_all();      // the previous piece has left the buffer
          __syncwarp();
          uint4 *dst = reinterpret_cast<uint4 *>(stg + lane * kP2EpiCols * 2);
#pragma unroll
          for (int j = 0; j < kP2EpiCols / 8; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            ptx::tma_store_2d(&tmY, stg, nt * kP2N + (kP2N / 2) * h + kP2EpiCols * pc, row0);
            ptx::bulk_commit();
          }
        }
        continue;
      }
      const int row = row0 + lane;
      if (row < g.M) {
        __nv_bfloat16 *yrow = g.Y + static_cast<int64_t>(row) * g.ldy;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            if (32 * c + 8 * v >= kP2N / 2) continue;           // the other half's columns
            const int n = nt * kP2N + (kP2N / 2) * h + 32 * c + 8 * v;
            if (g.y_vec && n + 8 <= g.N) {
              uint32_t pk[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[c][8 * v + 2 * i]),
                                                          __uint_as_float(r[c][8 * v + 2 * i + 1]));
                pk[i] = *reinterpret_cast<uint32_t *>(&b2);
              }
              *reinterpret_cast<uint4 *>(yrow + n) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                if (n + i < g.N) yrow[n + i] = __float2bfloat16_rn(__uint_as_float(r[c][8 * v + i]));
            }
          }
        }
      }
    }
  }

  // the tensor stores of Y are complete before the CTA leaves
  if (warp >= 2 && lane == 0) ptx::bulk_wait_all();
  if (warp == 0 && lane == 0) *issued_slot = it;
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();
  // Neither CTA issues a copy or an MMA past this point.  Before either
  // leaves, everything issued lands: the leader's commit arrives on both
  // CTAs' drain barriers once every MMA (and scale copy) has finished, and
  // the leader settles the pair's outstanding stages on its full barriers.
  // Stage i was issued by both producers, by one, or by none; only the last
  // kP2Stages stages can be outstanding (a producer issues stage i after the
  // MMAs consumed stage i - kP2Stages, which needed both halves).  Where one
  // half was never issued, the leader supplies its arrival and byte count
  // itself, so the phase completes when the other half lands.  On a normal
  // exit every stage is complete and each wait returns at once.
  if (warp == 1 && lane == 0) {
    if (leader) ptx::mma2_commit_both(drain);
    ptx::mbar_wait_cycles(drain, 0, kWaitLimit);
  }
  if (leader && warp == 0 && lane == 0) {
    const int L = it;
    const int P = static_cast<int>(ptx::ld_cluster_u32(ptx::map_to_rank(ptx::smem_addr(issued_slot), 1)));
    const int hi = max(L, P);
    for (int i = max(0, hi - kP2Stages); i < hi; ++i) {
      const int s = i % kP2Stages, k = i % n_iters;
      const bool wide = k < n16s;
      const int j0 = kP2Sub * (wide ? k : k - n16s);
      const int nsub = min(kP2Sub, (wide ? g.n16_stages : g.n8_stages) - j0);
      const uint32_t half = static_cast<uint32_t>(nsub) * ((wide ? bytes16 : bytes8) / 2);
      if (i < L && i >= P) {
        ptx::mbar_complete_tx(&full[s], half);
      } else if (i >= L && i < P) {
        ptx::mbar_arrive_expect_tx(&full[s], 2 * half);
        ptx::mbar_complete_tx(&full[s], half);
      }
      ptx::mbar_wait_cycles(&full[s], (i / kP2Stages) & 1, kWaitLimit);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc2(tmem, kTmemCols);
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
  int32_t tile_rows;    // rows per output tile: tile t's rows fill chunk rows 256 t .. 256 t + tile_rows - 1
};

// Item space of the staging kernel, one item per (operand, row, block):
// [wide A][wide B][4-bit A][4-bit B], each range starting at a multiple of 32
// items.  Wide items cover the 8- and 6-bit blocks of the real rows; 4-bit
// items cover the scale-chunk grid (rows padded to 128-row groups, blocks to
// 4-block k-groups), the padding items writing only their 2^0 scale byte.
struct StageArgs {
  StageOperand op[2];
  int32_t nb[3];        // blocks per segment
  int32_t nbw;          // wide blocks per row: nb[0] + nb[1]
  int32_t nb4p;         // 4-bit blocks per row padded to k-groups: nkg * 4
  int64_t k16, k4;
  int32_t nkg;          // k-groups of 4 blocks in the 4-bit segment
  int32_t start[5];     // item ranges (the last entry is the end)
  uint32_t nbw_magic, nb4p_magic;   // floor(2^32 / d) + 1 for the divisions i / d (0: divide)
};

// i / d by multiply-high with magic = floor(2^32 / d) + 1, exact while
// i * d < 2^32 (the host passes 0 when some item index breaks that).
__device__ __forceinline__ int div_magic(int i, int d, uint32_t magic) {
  return magic ? static_cast<int>(__umulhi(static_cast<uint32_t>(i), magic)) : i / d;
}

__device__ __forceinline__ int64_t sf_index(int64_t r, int64_t b, int32_t nrg) {
  return ((b >> 2) * nrg + (r >> 7)) * kSfChunk + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}


// 6/8-bit block -> 32 exact bf16 values q * 2^(e-m+2), as 16 packed words.
__device__ __forceinline__ void wide6_words_fast(const uint32_t (&w)[6], uint8_t sbyte, uint32_t (&pk)[16]);

template <int M>
__device__ __forceinline__ void wide_block_words(const uint8_t *c, uint8_t sbyte, uint32_t (&pk)[16]) {
  if constexpr (M == 6) {
    if (sbyte >= 13 && sbyte <= 251) {                     // 192 * step and the results are normal bf16
      const uint2 a = *reinterpret_cast<const uint2 *>(c), b = *reinterpret_cast<const uint2 *>(c + 8),
                  d = *reinterpret_cast<const uint2 *>(c + 16);
      const uint32_t w[6] = {a.x, a.y, b.x, b.y, d.x, d.y};
      wide6_words_fast(w, sbyte, pk);
      return;
    }
  }
  const float step = pow2f(static_cast<int>(sbyte) - 127 - M + 2);
  int q[kBlock];
  if constexpr (M == 8) {
    const uint4 a = *reinterpret_cast<const uint4 *>(c), b = *reinterpret_cast<const uint4 *>(c + 16);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int t = 0; t < kBlock; ++t) q[t] = static_cast<int>(static_cast<int8_t>((w[t >> 2] >> (8 * (t & 3))) & 0xFF));
  } else {
    const uint2 a = *reinterpret_cast<const uint2 *>(c), b = *reinterpret_cast<const uint2 *>(c + 8),
                d = *reinterpret_cast<const uint2 *>(c + 16);
    const uint32_t w[6] = {a.x, a.y, b.x, b.y, d.x, d.y};
#pragma unroll
    for (int t = 0; t < kBlock; ++t) {
      const int pos = 6 * t, word = pos >> 5, off = pos & 31;
      uint32_t f = w[word] >> off;
      if (off > 26) f |= w[word + 1] << (32 - off);
      q[t] = static_cast<int>(f << 26) >> 26;    // sign-extend the 6-bit field
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(code_to_float(q[2 * i]) * step, code_to_float(q[2 * i + 1]) * step);
    pk[i] = *reinterpret_cast<uint32_t *>(&h);
  }
}

// 6-bit block -> 32 exact bf16 values q * 2^(e-4) as 16 packed words, two
// codes per instruction: a code's 16-bit lane is made the bf16 of 192 + q
// (0x4320 + (f ^ 0x20) for the 6-bit field f; 192 + q stays in [128, 256),
// where bf16 integers are exact), then one packed fma (192+q)*s - 192*s
// gives q*s exactly (q*s is a bf16: <= 5 significant bits, exponent in range).
__device__ __forceinline__ void wide6_words_fast(const uint32_t (&w)[6], uint8_t sbyte, uint32_t (&pk)[16]) {
  const int e = static_cast<int>(sbyte) - 127 - 4;    // step 2^(e-m+2), m = 6
  // the step is >= 2^-131; below 2^-126 bf16 has no normal encoding: use the fp32 path
  const float step = pow2f(e);
  const __nv_bfloat162 s2 = __floats2bfloat162_rn(step, step);
  const __nv_bfloat162 c2 = __floats2bfloat162_rn(-192.f * step, -192.f * step);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    uint32_t f[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int pos = 6 * (2 * i + h), word = pos >> 5, off = pos & 31;
      uint32_t v = w[word] >> off;
      if (off > 26) v |= w[word + 1] << (32 - off);
      f[h] = v & 0x3Fu;
    }
    const uint32_t x = (f[0] | (f[1] << 16)) ^ 0x00200020u;
    const uint32_t b = x + 0x43204320u;
    const __nv_bfloat162 r = __hfma2(*reinterpret_cast<const __nv_bfloat162 *>(&b), s2, c2);
    pk[i] = *reinterpret_cast<const uint32_t *>(&r);
  }
}

// 32-byte store (one 256-bit access; p 32-byte aligned).
__device__ __forceinline__ void st_global_32B(void *p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// 6/8-bit block -> 32 exact bf16 values, two 32-byte stores.
template <int M>
__device__ __forceinline__ void stage_wide_block(const uint8_t *c, uint8_t sbyte, __nv_bfloat16 *dst) {
  uint32_t pk[16];
  wide_block_words<M>(c, sbyte, pk);
  const uint32_t lo[8] = {pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]};
  const uint32_t hi[8] = {pk[8], pk[9], pk[10], pk[11], pk[12], pk[13], pk[14], pk[15]};
  st_global_32B(dst, lo);
  st_global_32B(dst + 16, hi);
}

constexpr int kStageU = 2;   // 32-item groups per warp round of the staging kernel

// Eight 4-bit codes (one word, low nibble first) -> their eight E4M3 bytes
// (q/4), in register byte permutes: the code's low three bits pick entry
// n & 7 of an 8-byte table (t[0..1]: codes 0..7; t[2..3]: codes 8..15, the
// negative ones), and a third permute takes, byte by byte, the second
// table's pick where the code's bit 3 is set.
// Byte permute; every selector nibble here has bit 3 clear (a plain pick).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint2 e4m3_of_nibbles(uint32_t x, const uint32_t (&t)[4]) {
  const uint32_t lo3 = x & 0x77777777u;
  const uint32_t pick = ((x >> 1) & 0x44444444u) | 0x32103210u;   // byte j: j, or j + 4 when bit 3 is set
  const uint32_t p0 = prmt(t[0], t[1], lo3), n0 = prmt(t[2], t[3], lo3);
  const uint32_t p1 = prmt(t[0], t[1], lo3 >> 16), n1 = prmt(t[2], t[3], lo3 >> 16);
  return make_uint2(prmt(p0, n0, pick), prmt(p1, n1, pick >> 16));
}

// One thread per item, warps on consecutive items (consecutive blocks of a
// row), so code loads and converted stores are contiguous across the warp.
// 4-bit codes become E4M3 bytes by register byte permutes; a k-group's four
// scale bytes are gathered by shuffles and written as one word of the tensor
// core's 512-byte chunk layout.
__global__ void __launch_bounds__(256) gemm_stage_kernel(StageArgs a) {
  pdl_wait();
  pdl_trigger();
  // E4M3 of q/4 for the codes 0..15 (q = code, or code - 16 from 8 on), one
  // byte each: 0, .25, .5, .75, 1, 1.25, 1.5, 1.75, -2, -1.75, ..., -.25
  const uint32_t tab[4] = {0x34302800u, 0x3E3C3A38u, 0xBABCBEC0u, 0xA8B0B4B8u};
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  // a warp takes kStageU groups of 32 items per round: the 4-bit groups'
  // code and scale loads are all issued before any of them is converted
  for (int base = (blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * (32 * kStageU); base < a.start[4];
       base += nwarps * 32 * kStageU) {
    int rg[kStageU], row[kStageU], b[kStageU], real[kStageU];
    bool live[kStageU];
    uint4 v[kStageU];
    uint32_t sb[kStageU];
#pragma unroll
    for (int u = 0; u < kStageU; ++u) {
      const int gb = base + 32 * u;                    // this group's first item (uniform)
      rg[u] = 0;
      while (rg[u] < 4 && gb >= a.start[rg[u] + 1]) ++rg[u];
      sb[u] = 0x7Fu;                                   // 2^0 for padding rows and blocks
      live[u] = false;
      if (rg[u] >= 2 && rg[u] < 4) {
        const StageOperand &op = a.op[rg[u] & 1];
        const int i = gb + lane - a.start[rg[u]];
        row[u] = div_magic(i, a.nb4p, a.nb4p_magic);    // row of the chunk grid
        b[u] = i - row[u] * a.nb4p;
        const int lr = row[u] & 255;
        real[u] = (row[u] >> 8) * op.tile_rows + lr;   // the operand row it holds
        live[u] = lr < op.tile_rows && real[u] < op.rows && b[u] < a.nb[2];
        if (live[u]) {
          v[u] = *reinterpret_cast<const uint4 *>(op.codes[2] + real[u] * op.cpitch[2] + static_cast<int64_t>(b[u]) * 16);
          sb[u] = op.scales[2][real[u] * op.spitch[2] + b[u]];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kStageU; ++u) {
      if (rg[u] >= 4) break;                           // past the last range (uniform)
      const int gb = base + 32 * u;
      const StageOperand &op = a.op[rg[u] & 1];
      if (rg[u] < 2) {
        const int i = gb + lane - a.start[rg[u]];
        const int r = div_magic(i, a.nbw, a.nbw_magic), bw = i - r * a.nbw;
        if (r < op.rows) {
          const int g = bw < a.nb[0] ? 0 : 1;
          const int bb = g == 0 ? bw : bw - a.nb[0];
          const uint8_t sbyte = op.scales[g][r * op.spitch[g] + bb];
          __nv_bfloat16 *dst = op.x16 + static_cast<int64_t>(r) * a.k16 + static_cast<int64_t>(bw) * kBlock;
          if (g == 0) stage_wide_block<8>(op.codes[0] + r * op.cpitch[0] + static_cast<int64_t>(bb) * 32, sbyte, dst);
          else stage_wide_block<6>(op.codes[1] + r * op.cpitch[1] + static_cast<int64_t>(bb) * 24, sbyte, dst);
        }
      } else {
        if (live[u]) {
          const uint32_t in[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
          uint32_t out[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint2 e = e4m3_of_nibbles(in[j], tab);
            out[2 * j] = e.x;
            out[2 * j + 1] = e.y;
          }
          st_global_32B(op.x8 + static_cast<int64_t>(real[u]) * a.k4 + static_cast<int64_t>(b[u]) * kBlock, out);
        }
        // lanes 4j..4j+3 hold blocks 4k..4k+3 of one row (ranges and nb4p are multiples of 4)
        uint32_t w = sb[u];
        w |= __shfl_down_sync(0xffffffffu, w, 1) << 8;
        w |= __shfl_down_sync(0xffffffffu, w, 2) << 16;
        if ((lane & 3) == 0) *reinterpret_cast<uint32_t *>(op.sf + sf_index(row[u], b[u], op.nrg)) = w;
      }
    }
  }
}

constexpr int64_t kPairMinM = 512;   // from here the 2-CTA pair kernel

// ---------------------------------------------------------------- host side

struct WsPlan {
  int64_t k16, k4;
  int32_t nkg, nrg_a, nrg_b, b_tile_rows;
  size_t off_a16, off_b16, off_a8, off_b8, off_sfa, off_sfb, total;
};

static WsPlan plan_workspace(const mxs_mxtensor *A, const mxs_mxtensor *W) {
  WsPlan p{};
  const int64_t M = A->rows, N = W->rows;
  p.k16 = A->lay.seg[0].k_pad + A->lay.seg[1].k_pad;
  p.k4 = A->lay.seg[2].k_pad;
  p.nkg = static_cast<int32_t>((p.k4 + 127) / 128);
  p.nrg_a = static_cast<int32_t>((M + kBM - 1) / kBM);
  // B's scale chunks follow the output tiles: 256-row tiles (one CTA) or
  // 240-row tiles (2-CTA pairs), two 128-row chunks per tile
  p.b_tile_rows = M >= kPairMinM ? kP2N : kBN;
  p.nrg_b = static_cast<int32_t>((N + p.b_tile_rows - 1) / p.b_tile_rows * 2);
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

bool make_plain_map(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, int64_t cols,
                    int64_t rows, int64_t ld, int box_cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * esize)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int *device_status_word() {
  struct Entry {
    unsigned long long ctx;
    int *addr;
  };
  static Entry cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (!ctx || cache[dev].ctx != ctx || !cache[dev].addr) {
    // first use on this device, or its context was reset since: the
    // symbol's address belongs to the current context's module
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess || !p) return nullptr;
    cache[dev] = Entry{current_context_id(), static_cast<int *>(p)};
  }
  return cache[dev].addr;
}

// 2-D byte map with 128-byte rows, no swizzle: the scale-chunk arrays seen as
// rows of 128 bytes (a 512-byte chunk is 4 rows).
static bool make_rows_map(CUtensorMap *m, void *base, int64_t total_bytes, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(total_bytes / 128)};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
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
  if (cudaMemcpyFromSymbol(&st, g_status, sizeof(int)) != cudaSuccess) return MXS_ERR_CUDA;
  if (st != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
    return static_cast<mxs_status>(st);
  }
  return MXS_OK;
}

extern "C" mxs_status mxs_set_wait_limit(int64_t cycles) {
  const long long v = cycles <= 0 ? kWaitLimit : std::min<long long>(cycles, kWaitLimit);
  return cudaMemcpyToSymbol(g_wait_limit, &v, sizeof(v)) == cudaSuccess ? MXS_OK : MXS_ERR_CUDA;
}

extern "C" mxs_status mxs_gemm_workspace_bytes(const mxs_mxtensor *A, const mxs_mxtensor *W, size_t *bytes) {
  if (!bytes) return MXS_ERR_ARG;
  mxs_status st = gemm_check(A, W);
  if (st != MXS_OK) return st;
  *bytes = small_fits(A, W) ? 0 : plan_workspace(A, W).total;   // the decode path needs none
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
  if (small_fits(A, W)) return gemm_small(A, W, Y, ldy, cs);
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
    op.tile_rows = o ? p.b_tile_rows : 256;
  }
  for (int g = 0; g < 3; ++g) sa.nb[g] = static_cast<int32_t>(A->lay.seg[g].k_pad / kBlock);
  sa.nbw = sa.nb[0] + sa.nb[1];
  sa.nb4p = p.nkg * 4;
  sa.k16 = p.k16;
  sa.k4 = p.k4;
  sa.nkg = p.nkg;
  {
    const int64_t sizes[4] = {M * sa.nbw, N * sa.nbw, static_cast<int64_t>(p.nrg_a) * 128 * sa.nb4p,
                              static_cast<int64_t>(p.nrg_b) * 128 * sa.nb4p};
    int64_t at = 0;
    for (int r = 0; r < 4; ++r) {
      if (at >= INT32_MAX) return MXS_ERR_SHAPE;
      sa.start[r] = static_cast<int32_t>(at);
      at += round_up(sizes[r], 32);
    }
    if (at >= INT32_MAX) return MXS_ERR_SHAPE;
    sa.start[4] = static_cast<int32_t>(at);
  }
  {
    auto magic = [](int64_t d, int64_t imax) -> uint32_t {
      return d > 1 && imax * d < (1ll << 32) ? static_cast<uint32_t>((1ull << 32) / static_cast<uint64_t>(d) + 1) : 0u;
    };
    sa.nbw_magic = magic(sa.nbw, std::max(sa.start[2] - sa.start[0], 0));
    sa.nb4p_magic = magic(sa.nb4p, std::max(sa.start[4] - sa.start[2], 0));
  }
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int sgrid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((sa.start[4] + 255) / 256, static_cast<int64_t>(nsm) * 8)));
  // the staging kernel goes out right before the tensor-core kernel, after
  // every host step that can fail: a failed call launches nothing
  auto launch_stage = [&]() {
    launch_pdl(gemm_stage_kernel, dim3(sgrid), dim3(256), 0, cs, sa);
    count_launch();
  };

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
  const int32_t n16_stages = static_cast<int32_t>((p.k16 + 63) / 64);
  const int32_t n8_stages = static_cast<int32_t>((p.k4 + 127) / 128);
  const int32_t y_vec = aligned16(Y) && (ldy * 2) % 16 == 0;
  if (M >= kPairMinM) {
    CUtensorMap mSFA{}, mSFB{};
    if (p.k4 > 0) {
      if (!make_rows_map(&mSFA, base + p.off_sfa, static_cast<int64_t>(p.nkg) * p.nrg_a * kSfChunk, 4) ||
          !make_rows_map(&mSFB, base + p.off_sfb, static_cast<int64_t>(p.nkg) * p.nrg_b * kSfChunk, 8))
        return MXS_ERR_CUDA;
    }
    if (p.k16 > 0) {   // the pair kernel loads 120-row boxes of B
      if (!make_map(&mB16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base + p.off_b16, p.k16, N, kP2BRows)) return MXS_ERR_CUDA;
    }
    if (p.k4 > 0) {
      if (!make_map(&mB8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base + p.off_b8, p.k4, N, kP2BRows)) return MXS_ERR_CUDA;
    }
    P2Args pa{};
    pa.M = static_cast<int32_t>(M);
    pa.N = static_cast<int32_t>(N);
    pa.n16_stages = n16_stages;
    pa.n8_stages = n8_stages;
    pa.m_tiles = static_cast<int32_t>((M + 255) / 256);
    pa.n_tiles = static_cast<int32_t>((N + kP2N - 1) / kP2N);
    pa.nrg_a = p.nrg_a;
    pa.nrg_b = p.nrg_b;
    pa.Y = reinterpret_cast<__nv_bfloat16 *>(Y);
    pa.ldy = ldy;
    pa.y_vec = y_vec;
    CUtensorMap mY{};
    pa.y_tma = y_vec && make_plain_map(&mY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, N, M, ldy, kP2EpiCols, 32);
    if (!ensure_smem(gemm_tc2_kernel, kP2SmemBytes)) return MXS_ERR_CUDA;
    const int tiles = pa.m_tiles * pa.n_tiles;
    const int pairs = std::max(1, std::min(tiles, nsm / 2));
    launch_stage();
    launch_pdl(gemm_tc2_kernel, dim3(2 * pairs), dim3(kP2Threads), kP2SmemBytes, cs, mA16, mB16, mA8, mB8, mSFA, mSFB, mY,
               pa);
    count_launch();
    return cuda_status(cudaGetLastError());
  }
  GemmArgs ga{};
  ga.M = static_cast<int32_t>(M);
  ga.N = static_cast<int32_t>(N);
  ga.n16_stages = n16_stages;
  ga.n8_stages = n8_stages;
  ga.nrg_a = p.nrg_a;
  ga.nrg_b = p.nrg_b;
  ga.sfa = base + p.off_sfa;
  ga.sfb = base + p.off_sfb;
  ga.Y = reinterpret_cast<__nv_bfloat16 *>(Y);
  ga.ldy = ldy;
  ga.y_vec = y_vec;
  if (!ensure_smem(gemm_tc_kernel, kGemmSmemBytes)) return MXS_ERR_CUDA;
  dim3 grid(static_cast<unsigned>((N + kBN - 1) / kBN), static_cast<unsigned>((M + kBM - 1) / kBM));
  launch_stage();
  launch_pdl(gemm_tc_kernel, dim3(grid), dim3(kGemmThreads), kGemmSmemBytes, cs, mA16, mB16, mA8, mB8, ga);
  count_launch();
  return cuda_status(cudaGetLastError());
}
