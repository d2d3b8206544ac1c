// convert.cu -- a packed layer from its latent factors.
//
// Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models"
// (research.samsung.com blog), section 3, "Magnitude Balancing and Scale Extraction": for the
// continuous proxies Uh [d_out][r] and Vh [d_in][r],
//     eta = sqrt( ||Vh||_F / ||Uh||_F ),   U := eta Uh,   V := Vh / eta,
//     s1_i = mean |U_ik| over k,           s2_j = mean |V_jk| over k,
// and "Phase 3" packs sign(U), sign(V).  eta > 0, so sign(U) = sign(Uh): the signs are packed
// in the same pass that reads the latents for the statistics (one HBM pass per matrix).
//
// Pass 1 (one per matrix) is the pack kernel's warp-per-(row, 32 words) task, which also
// writes the task's fp64 sums of |v| and v^2 (fixed-order warp tree).  Pass 2, one block,
// adds each row's task sums in order, forms both norms with a fixed tree over the rows,
// then eta and the fp16 scales (round to nearest even).  Every sum has a fixed order:
// results are run-to-run identical.
#include "nq_common.cuh"

namespace nq {

__global__ void __launch_bounds__(256) pack_stats_kernel(const float* __restrict__ latent, int64_t rows, int64_t r,
                                                         int64_t ld_latent, uint32_t* __restrict__ packed,
                                                         int64_t ld_words, double* __restrict__ part) {
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
            for (int u = 0; u < 32; ++u) v[u] = (w0 + u < words) ? __ldcs(src + u * 32) : 0.0f;
        }
        // word u is the same in every lane; lane u keeps it (binary select on the lane bits)
        uint32_t b[32];
        double sa = 0.0, sq = 0.0;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            b[u] = __ballot_sync(0xffffffffu, v[u] >= 0.0f);  // NaN >= 0 is false
            const double d = static_cast<double>(v[u]);
            sa += fabs(d);
            sq += d * d;
        }
#pragma unroll
        for (int lvl = 0, n = 16; lvl < 5; ++lvl, n >>= 1) {
            const bool hi = (lane >> lvl) & 1;
#pragma unroll
            for (int i = 0; i < n; ++i) b[i] = hi ? b[2 * i + 1] : b[2 * i];
        }
        const uint32_t mine = b[0];
        for (int off = 16; off > 0; off >>= 1) {
            sa += __shfl_xor_sync(0xffffffffu, sa, off);
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
        }
        const int64_t w = w0 + lane;
        if (w < ld_words) packed[row * ld_words + w] = (w < words) ? mine : 0u;
        if (lane == 0) {
            part[2 * task] = sa;
            part[2 * task + 1] = sq;
        }
    }
}

constexpr int kFinishThreads = 1024;

// Sum over the rows [0, rows) of a row quantity, each thread a strided subset in order, then
// a fixed tree over the block; every thread gets the total.
__device__ double block_rows_sum(const double* part, int64_t rows, int64_t tpr, int comp, double* scratch) {
    double acc = 0.0;
    for (int64_t i = threadIdx.x; i < rows; i += kFinishThreads) {
        double row = 0.0;
        for (int64_t t = 0; t < tpr; ++t) row += part[2 * (i * tpr + t) + comp];
        acc += row;
    }
    scratch[threadIdx.x] = acc;
    __syncthreads();
    for (int s = kFinishThreads / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) scratch[threadIdx.x] += scratch[threadIdx.x + s];
        __syncthreads();
    }
    const double tot = scratch[0];
    __syncthreads();
    return tot;
}

__global__ void __launch_bounds__(kFinishThreads) finish_scales_kernel(const double* __restrict__ part_u,
                                                                       int64_t d_out, int64_t tpr_u,
                                                                       const double* __restrict__ part_v,
                                                                       int64_t d_in, int64_t tpr_v, int64_t r,
                                                                       uint16_t* __restrict__ s1,
                                                                       uint16_t* __restrict__ s2, double* eta_out) {
    __shared__ double scratch[kFinishThreads];
    pdl_wait();
    const double su = block_rows_sum(part_u, d_out, tpr_u, 1, scratch);
    const double sv = block_rows_sum(part_v, d_in, tpr_v, 1, scratch);
    const double nu = sqrt(su), nv = sqrt(sv);
    const double eta = (nu > 0.0 && nv > 0.0) ? sqrt(nv / nu) : 1.0;
    if (threadIdx.x == 0 && eta_out) *eta_out = eta;
    const double inv_r = 1.0 / static_cast<double>(r);
    for (int64_t i = threadIdx.x; i < d_out; i += kFinishThreads) {
        double a = 0.0;
        for (int64_t t = 0; t < tpr_u; ++t) a += part_u[2 * (i * tpr_u + t)];
        s1[i] = __half_as_ushort(__double2half(eta * a * inv_r));
    }
    for (int64_t j = threadIdx.x; j < d_in; j += kFinishThreads) {
        double a = 0.0;
        for (int64_t t = 0; t < tpr_v; ++t) a += part_v[2 * (j * tpr_v + t)];
        s2[j] = __half_as_ushort(__double2half(a / eta * inv_r));
    }
}

}  // namespace nq

namespace {

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
int64_t tasks_per_row(int64_t ld_words) { return (ld_words + 31) / 32; }

nq_status launch_pack_stats(const float* latent, int64_t rows, int64_t r, int64_t ld_latent, uint32_t* packed,
                            int64_t ld_words, double* part, cudaStream_t stream) {
    const int64_t tasks = rows * tasks_per_row(ld_words);
    if (tasks == 0) return NQ_OK;
    const int threads = 256;
    int64_t blocks = (tasks + threads / 32 - 1) / (threads / 32);
    const int64_t cap = static_cast<int64_t>(nq_host::sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    nq::pack_stats_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(latent, rows, r, ld_latent, packed,
                                                                                ld_words, part);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_LAUNCH;
}

}  // namespace

size_t nq_from_latent_ws(int64_t d_out, int64_t d_in, int64_t ldu, int64_t ldv) {
    return align256(static_cast<size_t>(d_out * tasks_per_row(ldu)) * 16) +
           align256(static_cast<size_t>(d_in * tasks_per_row(ldv)) * 16);
}

nq_status nq_launch_from_latent(const float* Uh, int64_t ld_uh, const float* Vh, int64_t ld_vh, int64_t d_out,
                                int64_t d_in, int64_t r, uint32_t* U, int64_t ldu, uint32_t* V, int64_t ldv,
                                uint16_t* s1, uint16_t* s2, double* eta, void* ws, cudaStream_t stream) {
    double* part_u = static_cast<double*>(ws);
    double* part_v = reinterpret_cast<double*>(static_cast<char*>(ws) +
                                               align256(static_cast<size_t>(d_out * tasks_per_row(ldu)) * 16));
    nq_status st = launch_pack_stats(Uh, d_out, r, ld_uh, U, ldu, part_u, stream);
    if (st != NQ_OK) return st;
    if ((st = launch_pack_stats(Vh, d_in, r, ld_vh, V, ldv, part_v, stream)) != NQ_OK) return st;
    int64_t tpr_u = tasks_per_row(ldu), tpr_v = tasks_per_row(ldv);
    void* args[] = {&part_u, &d_out, &tpr_u, &part_v, &d_in, &tpr_v, &r, &s1, &s2, &eta};
    return nq_host::launch_pdl(reinterpret_cast<const void*>(nq::finish_scales_kernel), dim3(1),
                               dim3(nq::kFinishThreads), 0, stream, args, false) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_LAUNCH;
}
