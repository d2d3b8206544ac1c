// pack.cu -- sign extraction + bit packing of latent fp32 factors.
//
// Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models"
// (research.samsung.com blog), section 3, "Step 3: Factorized Component Refinement": the
// binary factors are sign(U), sign(V) of latent matrices; "Phase 3": the frozen signs are
// packed into integer formats.  Bit (i, k) = (latent[i][k] >= 0), word k/32, bit k%32.
//
// HBM-bound stream: each warp owns 32 consecutive output words of one row (1024 latent
// values).  For each of those words the 32 lanes read 32 consecutive floats (one 128-byte
// coalesced transaction) and __ballot_sync turns the 32 comparisons into the word, lane l
// supplying bit l -- exactly the LSB-first order.  Lane u keeps word u (picked from the 32
// warp-uniform ballots by a binary select on its lane bits), so the 32 words leave in one
// coalesced 128-byte store.  All 32 loads of a warp are independent and are issued back to
// back, keeping enough bytes in flight to cover DRAM latency; full tasks skip the bounds
// checks.  The ALU work per bit is what bounds a naive version of this loop, not HBM.
#include "nq_common.cuh"

namespace nq {

__global__ void __launch_bounds__(256) pack_signs_kernel(const float* __restrict__ latent, int64_t rows,
                                                           int64_t r, int64_t ld_latent,
                                                           uint32_t* __restrict__ packed, int64_t ld_words) {
    const int lane = threadIdx.x & 31;
    const int64_t words = r / 32;
    const int64_t tasks_per_row = (ld_words + 31) / 32;
    const int64_t n_tasks = rows * tasks_per_row;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;

    for (int64_t task = warp; task < n_tasks; task += n_warps) {
        const int64_t row = task / tasks_per_row;
        const int64_t w0 = (task - row * tasks_per_row) * 32;
        const float* src = latent + row * ld_latent + w0 * 32 + lane;
        float v[32];
        if (w0 + 32 <= words) {  // a full task: no bounds to check
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = __ldcs(src + u * 32);
        } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                // words past r/32 are padding: nothing is read for them
                v[u] = (w0 + u < words) ? __ldcs(src + u * 32) : -1.0f;
            }
        }
        // word u is the same in every lane; lane u keeps it, picked by a binary select on the
        // bits of the lane index (31 selects instead of 32 compare-and-selects)
        uint32_t b[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) b[u] = __ballot_sync(0xffffffffu, v[u] >= 0.0f);  // NaN >= 0 is false
#pragma unroll
        for (int lvl = 0, n = 16; lvl < 5; ++lvl, n >>= 1) {
            const bool hi = (lane >> lvl) & 1;
#pragma unroll
            for (int i = 0; i < n; ++i) b[i] = hi ? b[2 * i + 1] : b[2 * i];
        }
        const uint32_t mine = b[0];
        const int64_t w = w0 + lane;
        if (w < ld_words) packed[row * ld_words + w] = (w < words) ? mine : 0u;
    }
}

}  // namespace nq

// ------------------------------------------------------------------------------ host side
nq_status nq_launch_pack(const float* latent, int64_t rows, int64_t r, int64_t ld_latent, uint32_t* packed,
                         int64_t ld_words, cudaStream_t stream) {
    const int64_t tasks = rows * ((ld_words + 31) / 32);
    if (tasks == 0) return NQ_OK;
    const int threads = 256;
    const int64_t warps_per_block = threads / 32;
    int64_t blocks = (tasks + warps_per_block - 1) / warps_per_block;
    const int64_t cap = static_cast<int64_t>(nq_host::sm_count()) * 8;  // 8 blocks (64 warps) per SM
    if (blocks > cap) blocks = cap;
    nq::pack_signs_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(latent, rows, r, ld_latent,
                                                                                packed, ld_words);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_LAUNCH;
}
