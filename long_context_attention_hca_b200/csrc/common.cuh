// common.cuh -- shared device/host helpers of the sm_100a kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/hca.h"

namespace hca {

// Records the last CUDA error for hca_last_cuda_error().
void set_last_cuda_error(int e);

#define HCA_CHECK_LAUNCH()                                   \
    do {                                                     \
        cudaError_t _e = cudaGetLastError();                 \
        if (_e != cudaSuccess) {                             \
            ::hca::set_last_cuda_error((int)_e);             \
            return HCA_ERR_CUDA;                             \
        }                                                    \
    } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Number of SMs of the current device (queried once per process and device).
int sm_count();
// process-wide CTA cap of a decode attention launch (0: none); see hca_set_launch_budget
int launch_budget(int op);
// Sets this thread's override of a launch budget (0: none); returns the previous one.
int thread_budget_swap(int op, int max_ctas);
// process-wide: sparse decode attention reads its query before waiting on the previous kernel; see hca_set_early_query
int early_query();
// default CTA cap of the dense decode attention beside the decode select of B rows (topk.cu)
int dense_beside_select(int B);

// Programmatic dependent launch.  A kernel launched by launch_pdl may be
// scheduled while the previous kernel of its stream is still running; it calls
// pdl_wait() before it reads anything that kernel (or any earlier work) wrote:
// the wait returns once the previous kernel has completed and its stores are
// visible (for a normal launch it returns at once).  pdl_trigger() in the
// previous kernel lets the dependent one be scheduled before its own CTAs exit.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- device
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// Two e4m3fn values (fp32 in) -> packed bytes (lo in bits 0..7, hi in 8..15),
// round to nearest even, saturating to +-448 (cvt ... .satfinite).
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two e4m3fn bytes (lo in bits 0..7) -> f16x2 (exact: every e4m3 value is an fp16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
    return r;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t v) {
    __half2 h = *reinterpret_cast<__half2*>(&v);
    return __half22float2(h);
}

}  // namespace hca
