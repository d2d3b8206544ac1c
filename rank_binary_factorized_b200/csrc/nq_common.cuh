// nq_common.cuh -- device-side helpers shared by the libnq kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nq.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "libnq is written for sm_100a (B200) only"
#endif

// Every workspace starts with this many reserved bytes, which the kernels neither read nor
// write; the per-call scratch follows.
#define NQ_WS_HEADER_BYTES 4096
#define NQ_MAX_RANK NQ_MAX_RANK_LIMIT

namespace nq {

// Device error word (one per device that loads the library, defined in api.cu; kernels get
// its address as an argument).  Set with atomicOr by a kernel whose bounded wait gave up,
// read and cleared by nq_sync_status.
constexpr unsigned int kErrTimeout = 1u;

// Iteration cap for every spin-wait on device (each iteration sleeps ~128 ns with
// __nanosleep after the first few polls; 2^22 polls is well over a second).
constexpr unsigned int kSpinLimit = 1u << 22;

__device__ __forceinline__ void flag_error(unsigned int* word, unsigned int bits) { atomicOr(word, bits); }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float f16_bits_to_float(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

// fp32 -> bf16, round to nearest even (the CUDA intrinsic).
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Programmatic dependent launch: wait for the grid queued before this one to finish and
// publish its memory, and let the next grid start its prologue.  Both are no-ops when the
// kernel was launched without the programmatic-serialisation attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace nq

// Host-side launch plumbing shared by the translation units (defined in api.cu).
namespace nq_host {
bool pdl_on();                                    // programmatic dependent launch (off: NQ_DISABLE_PDL=1)
// Validation shared by the decode entry points: the layer, 1 <= M <= NQ_MATVEC_MAX_M and the
// shared memory stage 2 needs.  NQ_OK or the status the entry point returns.
nq_status check_decode_call(const nq_lrb_layer* L, int64_t M);
bool device_ready();                              // current device is sm_100 and set up
int sm_count();                                   // multiprocessors of the current device
unsigned int* error_word();                       // device address of the error word
cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s, void** args,
                       bool pdl);
// as launch_pdl, with thread-block clusters of (1, cluster_y, 1) when cluster_y > 1
cudaError_t launch_ex(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s, void** args, bool pdl,
                      int cluster_y);
}  // namespace nq_host

// Decode path (decode.cu): y = layer(x) for M <= NQ_MATVEC_MAX_M; with grad != nullptr it
// writes grad[i] = sum_m cot[m][i] (U t_m)_i (the s1-gradient of sum_m <cot_m, y_m>) instead
// of y.
nq_status nq_launch_decode(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                           cudaStream_t stream, bool pdl, const uint16_t* cot = nullptr, float* grad = nullptr);
// Decode path for n <= 4 projections sharing x, one launch per stage (decode.cu).
nq_status nq_launch_decode_group(const nq_lrb_layer* const* Ls, int n, const uint16_t* x, uint16_t* const* ys,
                                 int64_t M, void* ws, cudaStream_t stream, bool pdl, const uint16_t* cot = nullptr,
                                 float* grad = nullptr);
size_t nq_decode_group_workspace_bytes(const nq_lrb_layer* const* Ls, int n, int64_t M);
// Prefill path (prefill.cu): Y = layer(x) on the tensor cores; with grad != nullptr it writes
// grad[i] = sum_m cot[m][i] (T U^T)[m][i] instead of Y.
nq_status nq_launch_prefill(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                            cudaStream_t stream, bool pdl, const uint16_t* cot = nullptr, float* grad = nullptr);
// GEMM 1 alone (prefill.cu): Z = fp16(x . s2) and T = fp16(Z V) into the workspace at the
// offsets nq_prefill_stage1_layout gives (bytes = the extent of the region).
void nq_prefill_stage1_layout(const nq_lrb_layer* L, int64_t M, size_t* off_z, int64_t* ldz, size_t* off_t,
                              int64_t* ldt, size_t* bytes);
nq_status nq_launch_prefill_stage1(const nq_lrb_layer* L, const uint16_t* x, int64_t M, void* ws, cudaStream_t stream,
                                   bool pdl);
// Stage 1 alone (decode.cu): t = V^T (s2 . x) [M][r] fp32 into t, M <= NQ_MATVEC_MAX_M.
nq_status nq_launch_decode_stage1(const nq_lrb_layer* L, const uint16_t* x, int64_t M, float* t, cudaStream_t stream,
                                  bool pdl);
// Stage 1 alone for two layers with their own inputs, one launch (decode.cu).
nq_status nq_launch_decode_stage1_pair(const nq_lrb_layer* L0, const uint16_t* x0, float* t0, const nq_lrb_layer* L1,
                                       const uint16_t* x1, float* t1, int64_t M, cudaStream_t stream, bool pdl);
