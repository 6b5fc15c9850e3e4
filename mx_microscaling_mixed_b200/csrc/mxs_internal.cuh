// mxs_internal.cuh -- shared helpers of libmxs (host checks, launch
// accounting, small PTX wrappers).  Device code here is sm_100a only.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "mxs.h"

namespace mxs {

constexpr int kBlock = 32;          // MXINT block length
constexpr int kSegBits[3] = {8, 6, 4};
// Width of segment g (order 8, 6, 4) in host or device code.
__host__ __device__ constexpr int seg_bits(int g) { return g == 0 ? 8 : (g == 1 ? 6 : 4); }

// Kernels launched by this library (for the caller's accounting).
void count_launch(int n = 1);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
__host__ __device__ inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
__host__ __device__ inline int64_t pad32(int64_t n) { return round_up(n, kBlock); }

// Bytes of one packed row of a segment of k_pad positions at `bits`.
inline int64_t seg_row_bytes(int64_t k_pad, int bits) { return k_pad * bits / 8; }

inline size_t dtype_size(mxs_dtype t) { return t == MXS_F32 ? 4 : 2; }
inline bool dtype_ok(mxs_dtype t) { return t == MXS_F32 || t == MXS_BF16; }

// Checks that the current device is a compute-capability 10.x part.
mxs_status check_device();

// Unique id of the CUDA context current on this thread (the driver's
// context id, unique for the life of the process), or 0 when no context is
// current yet.  Per-device caches of device addresses and kernel attributes
// are keyed by it, so that a device reset (which destroys the context and
// with it every module's device addresses) invalidates them.
unsigned long long current_context_id();

// Validates a layout against its own invariants (host only).
mxs_status check_layout(const mxs_layout *lay);

// Validates a quantised tensor's pointers and pitches (host only).
mxs_status check_mxtensor(const mxs_mxtensor *t);

inline mxs_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MXS_OK : MXS_ERR_CUDA; }

// Raises a kernel's dynamic shared memory limit to at least `bytes`, once
// per (kernel, device): the attribute belongs to the kernel on the current
// device.
bool ensure_smem_impl(const void *kernel, int bytes);
template <typename Kernel>
inline bool ensure_smem(Kernel k, int bytes) {
  return ensure_smem_impl(reinterpret_cast<const void *>(k), bytes);
}

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialisation and calls pdl_trigger() at its
// start, so the next kernel in the stream may be scheduled once every CTA
// of this one is running (none of this grid is still waiting for an SM, so
// the early CTAs take only resources this grid does not need).  Before its
// first access to global memory, each kernel calls pdl_wait(), which
// returns once the previous kernel has completed and its memory operations
// are visible; only setup that touches no global memory (barriers, tensor
// memory, descriptor prefetch) may come before it.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- device side
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Value of an integer |q| < 2^22 as an exact float: the integer rides in the
// mantissa of 1.5*2^23 and is taken back out by a subtraction.
__device__ __forceinline__ float code_to_float(int q) {
  return __uint_as_float(static_cast<uint32_t>(0x4B400000 + q)) - 12582912.0f;
}

// Exact x * 2^k for the exponents the MXINT coder needs (k in [-126, 140]).
// A single multiply by a normal power of two is exact unless the result is
// subnormal, which only happens for values that round to code 0 anyway.
__device__ __forceinline__ float scale_pow2(float x, int k) {
  if (k > 127) {
    x *= __uint_as_float(static_cast<uint32_t>(64 + 127) << 23);
    k -= 64;
  }
  return x * __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
}

// Exact value 2^k as a float for k in [-149, 127] (subnormal below -126).
__device__ __forceinline__ float pow2f(int k) {
  return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23)
                   : __uint_as_float(1u << (k + 149));
}

}  // namespace mxs
