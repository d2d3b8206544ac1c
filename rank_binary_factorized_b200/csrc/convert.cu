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
// writes the task's fp64 sums of |v| and v^2 (fixed-order warp tree).  Pass 2, one thread per
// row, adds each row's task sums in order and reduces the squares per block by a fixed tree.
// Pass 3: every block forms both norms from the block partials (fixed order), then eta and
// the fp16 scales of its rows (round to nearest even).  Every sum has a fixed order: results
// are run-to-run identical.
#include <algorithm>

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

constexpr int kRowThreads = 256;  // rows per block of the two finishing kernels

// Fixed tree over the block's kRowThreads values in sh (every thread returns the total).
__device__ double block_tree_sum(double v, double* sh) {
    sh[threadIdx.x] = v;
    __syncthreads();
    for (int s = kRowThreads / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) sh[threadIdx.x] += sh[threadIdx.x + s];
        __syncthreads();
    }
    const double tot = sh[0];
    __syncthreads();
    return tot;
}

// Pass 2: one thread per row (blocks [0, bu) take the rows of U, the rest the rows of V):
// rowabs[i] = sum over the row's tasks, in order, of the task's sum |v|, and per block the sum
// of its rows' sums v^2 by a fixed tree, blockq[b].
__global__ void __launch_bounds__(kRowThreads) row_stats_kernel(const double* __restrict__ part_u, int64_t d_out,
                                                              int64_t tpr_u, const double* __restrict__ part_v,
                                                              int64_t d_in, int64_t tpr_v, int bu,
                                                              double* __restrict__ rowabs_u,
                                                              double* __restrict__ rowabs_v,
                                                              double* __restrict__ blockq) {
    __shared__ double sh[kRowThreads];
    pdl_wait();
    const bool is_u = static_cast<int>(blockIdx.x) < bu;
    const int64_t i = static_cast<int64_t>(is_u ? blockIdx.x : blockIdx.x - bu) * kRowThreads + threadIdx.x;
    const int64_t rows = is_u ? d_out : d_in, tpr = is_u ? tpr_u : tpr_v;
    const double* part = is_u ? part_u : part_v;
    double a = 0.0, q = 0.0;
    if (i < rows) {
        for (int64_t t = 0; t < tpr; ++t) {
            a += part[2 * (i * tpr + t)];
            q += part[2 * (i * tpr + t) + 1];
        }
        (is_u ? rowabs_u : rowabs_v)[i] = a;
    }
    const double tot = block_tree_sum(q, sh);
    if (threadIdx.x == 0) blockq[blockIdx.x] = tot;
}

// Sum of n block partials: thread t adds entries t, t + kRowThreads, ... in order, then a
// fixed tree.  Every block of the scales kernel computes the same value the same way.
__device__ double partials_sum(const double* p, int n, double* sh) {
    double acc = 0.0;
    for (int e = threadIdx.x; e < n; e += kRowThreads) acc += p[e];
    return block_tree_sum(acc, sh);
}

// Pass 3: eta from the two norms, then the fp16 scales of a grid-stride set of rows
// (rows of U first, then rows of V).
__global__ void __launch_bounds__(kRowThreads) scales_kernel(const double* __restrict__ rowabs_u, int64_t d_out,
                                                           const double* __restrict__ rowabs_v, int64_t d_in,
                                                           const double* __restrict__ blockq, int bu, int bv,
                                                           int64_t r, uint16_t* __restrict__ s1,
                                                           uint16_t* __restrict__ s2, double* eta_out) {
    __shared__ double sh[kRowThreads];
    pdl_wait();
    const double nu = sqrt(partials_sum(blockq, bu, sh));
    const double nv = sqrt(partials_sum(blockq + bu, bv, sh));
    const double eta = (nu > 0.0 && nv > 0.0) ? sqrt(nv / nu) : 1.0;
    if (blockIdx.x == 0 && threadIdx.x == 0 && eta_out) *eta_out = eta;
    const double inv_r = 1.0 / static_cast<double>(r);
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * kRowThreads + threadIdx.x; e < d_out + d_in;
         e += static_cast<int64_t>(gridDim.x) * kRowThreads) {
        if (e < d_out) s1[e] = __half_as_ushort(__double2half(eta * rowabs_u[e] * inv_r));
        else s2[e - d_out] = __half_as_ushort(__double2half(rowabs_v[e - d_out] / eta * inv_r));
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

// Workspace: task partials of U and V, then the row sums |.| of U and V, then the block
// partials of the squared norms.
struct ConvertLayout {
    size_t part_v, rowabs_u, rowabs_v, blockq, total;
    int bu, bv;
};

ConvertLayout convert_layout(int64_t d_out, int64_t d_in, int64_t ldu, int64_t ldv) {
    ConvertLayout c{};
    c.bu = static_cast<int>((d_out + nq::kRowThreads - 1) / nq::kRowThreads);
    c.bv = static_cast<int>((d_in + nq::kRowThreads - 1) / nq::kRowThreads);
    c.part_v = align256(static_cast<size_t>(d_out * tasks_per_row(ldu)) * 16);
    c.rowabs_u = c.part_v + align256(static_cast<size_t>(d_in * tasks_per_row(ldv)) * 16);
    c.rowabs_v = c.rowabs_u + align256(static_cast<size_t>(d_out) * 8);
    c.blockq = c.rowabs_v + align256(static_cast<size_t>(d_in) * 8);
    c.total = c.blockq + align256(static_cast<size_t>(c.bu + c.bv) * 8);
    return c;
}

size_t nq_from_latent_ws(int64_t d_out, int64_t d_in, int64_t ldu, int64_t ldv) {
    return convert_layout(d_out, d_in, ldu, ldv).total;
}

nq_status nq_launch_from_latent(const float* Uh, int64_t ld_uh, const float* Vh, int64_t ld_vh, int64_t d_out,
                                int64_t d_in, int64_t r, uint32_t* U, int64_t ldu, uint32_t* V, int64_t ldv,
                                uint16_t* s1, uint16_t* s2, double* eta, void* ws, cudaStream_t stream) {
    const ConvertLayout c = convert_layout(d_out, d_in, ldu, ldv);
    char* w = static_cast<char*>(ws);
    double* part_u = reinterpret_cast<double*>(w);
    double* part_v = reinterpret_cast<double*>(w + c.part_v);
    double* rowabs_u = reinterpret_cast<double*>(w + c.rowabs_u);
    double* rowabs_v = reinterpret_cast<double*>(w + c.rowabs_v);
    double* blockq = reinterpret_cast<double*>(w + c.blockq);
    nq_status st = launch_pack_stats(Uh, d_out, r, ld_uh, U, ldu, part_u, stream);
    if (st != NQ_OK) return st;
    if ((st = launch_pack_stats(Vh, d_in, r, ld_vh, V, ldv, part_v, stream)) != NQ_OK) return st;
    int64_t tpr_u = tasks_per_row(ldu), tpr_v = tasks_per_row(ldv);
    int bu = c.bu, bv = c.bv;
    {
        void* args[] = {&part_u, &d_out, &tpr_u, &part_v, &d_in, &tpr_v, &bu, &rowabs_u, &rowabs_v, &blockq};
        if (nq_host::launch_pdl(reinterpret_cast<const void*>(nq::row_stats_kernel), dim3(bu + bv),
                                dim3(nq::kRowThreads), 0, stream, args, false) != cudaSuccess)
            return NQ_ERR_LAUNCH;
    }
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(bu + bv, 2LL * nq_host::sm_count()));
    void* args[] = {&rowabs_u, &d_out, &rowabs_v, &d_in, &blockq, &bu, &bv, &r, &s1, &s2, &eta};
    return nq_host::launch_pdl(reinterpret_cast<const void*>(nq::scales_kernel), dim3(grid), dim3(nq::kRowThreads),
                               0, stream, args, true) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_LAUNCH;
}
