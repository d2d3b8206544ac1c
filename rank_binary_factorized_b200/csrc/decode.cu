// decode.cu -- batch 1..8 ("token-by-token") path of the LRB matmul.
//
// Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models"
// (research.samsung.com blog), section 2, factorisation equation, evaluated right to left
// straight from the packed signs; section 4, "Inference Performance", names this binary
// GEMV for decoding.
//
//   stage 1:  t[m][k] = sum_j V_jk * (s2_j * x[m][j])          (reduction over d_in)
//   stage 2:  y[m][i] = bf16( s1_i * sum_k U_ik * t[m][k] )      (reduction over r)
//
// Stage 1 is a split-d_in reduction: block (c, s) owns word chunk c (WC words = WC*32
// columns of t) and row slice s of V.  Threads own (word, bit group, row subset) and keep
// fp32 accumulators; the block folds its row subsets through shared memory, writes one
// partial per slice, and the last block of each chunk to finish (an atomic ticket) sums the
// partials in slice order.  No atomics touch the values, so t is run-to-run identical.
//
// Stage 2 stages t in shared memory transposed so that lanes reading consecutive words hit
// consecutive banks; each warp sweeps one row of U with 128-byte coalesced loads.
#include "nq_common.cuh"

namespace nq {

constexpr int kS1Threads = 256;
constexpr int kS1WordsPerChunk = 8;  // 32-byte row segments: one full DRAM sector per row

template <int MB>
struct S1Cfg {
    static constexpr int KB = (MB <= 2) ? 32 : (MB <= 4 ? 16 : 8);  // bits per thread
    static constexpr int NBG = 32 / KB;                                // bit groups per word
    static constexpr int JG = kS1Threads / (kS1WordsPerChunk * NBG);   // row subsets per block
    static constexpr int OUT = kS1WordsPerChunk * 32 * MB;             // outputs per block
};

__host__ __device__ __forceinline__ constexpr int pad32(int o) { return o + (o >> 5); }

template <int MB>
__global__ void __launch_bounds__(kS1Threads) decode_stage1_kernel(
    const uint32_t* __restrict__ V, int64_t ldv, const uint16_t* __restrict__ s2, const uint16_t* __restrict__ x,
    int M, int64_t d_in, int64_t r, int rows_per_slice, float* __restrict__ part, float* __restrict__ t,
    unsigned int* __restrict__ tickets) {
    using C = S1Cfg<MB>;
    extern __shared__ float smem[];
    float* z_s = smem;                             // [MB][rows_per_slice]
    float* red = smem + MB * rows_per_slice;       // [JG][pad32(OUT)]
    __shared__ unsigned int s_is_last;

    const int tid = threadIdx.x;
    const int wl = tid % kS1WordsPerChunk;
    const int bg = (tid / kS1WordsPerChunk) % C::NBG;
    const int jg = tid / (kS1WordsPerChunk * C::NBG);
    const int64_t nw = r / 32;
    const int64_t w = static_cast<int64_t>(blockIdx.x) * kS1WordsPerChunk + wl;
    const bool wvalid = w < nw;
    const int S = gridDim.y;
    const int s = blockIdx.y;
    const int64_t j0 = static_cast<int64_t>(s) * rows_per_slice;
    const int64_t j1 = min(d_in, j0 + rows_per_slice);
    const int rows = static_cast<int>(j1 - j0);

    pdl_wait();  // x (and the workspace) may be written by the previous grid

    // z[m][j] = s2_j * x[m][j] in fp32 (exact: 11 x 8 significant bits)
    for (int e = tid; e < MB * rows; e += kS1Threads) {
        const int m = e / rows;
        const int jj = e - m * rows;
        float z = 0.0f;
        if (m < M) z = f16_bits_to_float(s2[j0 + jj]) * bf16_bits_to_float(x[static_cast<int64_t>(m) * d_in + j0 + jj]);
        z_s[m * rows_per_slice + jj] = z;
    }
    __syncthreads();

    float acc[C::KB][MB];
#pragma unroll
    for (int c = 0; c < C::KB; ++c)
#pragma unroll
        for (int m = 0; m < MB; ++m) acc[c][m] = 0.0f;

    if (wvalid) {
        const uint32_t* vp = V + w;
        for (int jj = jg; jj < rows; jj += C::JG) {
            const uint32_t word = __ldg(vp + (j0 + jj) * ldv) >> (bg * C::KB);
            float z[MB];
#pragma unroll
            for (int m = 0; m < MB; ++m) z[m] = z_s[m * rows_per_slice + jj];
#pragma unroll
            for (int c = 0; c < C::KB; ++c) {
                // bit 1 -> +z, bit 0 -> -z: flip the sign bit of z when the bit is clear
                const uint32_t flip = ((~word) << (31 - c)) & 0x80000000u;
#pragma unroll
                for (int m = 0; m < MB; ++m) acc[c][m] += __uint_as_float(__float_as_uint(z[m]) ^ flip);
            }
        }
    }

    // fold the JG row subsets of this block
    {
        float* dst = red + jg * pad32(C::OUT);
#pragma unroll
        for (int c = 0; c < C::KB; ++c)
#pragma unroll
            for (int m = 0; m < MB; ++m) dst[pad32((wl * 32 + bg * C::KB + c) * MB + m)] = acc[c][m];
    }
    __syncthreads();

    const int64_t kbase = static_cast<int64_t>(blockIdx.x) * kS1WordsPerChunk * 32;
    for (int o = tid; o < C::OUT; o += kS1Threads) {
        float v = 0.0f;
        for (int g = 0; g < C::JG; ++g) v += red[g * pad32(C::OUT) + pad32(o)];
        const int m = o % MB;
        const int64_t k = kbase + o / MB;
        if (m < M && k < r) part[(static_cast<int64_t>(s) * M + m) * r + k] = v;
    }

    // last block of this chunk sums the S partials in slice order
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned int prev = atomicAdd(&tickets[blockIdx.x], 1u);
        s_is_last = (prev == static_cast<unsigned int>(S - 1)) ? 1u : 0u;
    }
    __syncthreads();
    if (s_is_last) {
        __threadfence();
        for (int o = tid; o < C::OUT; o += kS1Threads) {
            const int m = o % MB;
            const int64_t k = kbase + o / MB;
            if (m < M && k < r) {
                // fixed slice order; the loads of a group of 8 are independent and in flight together
                const float* pp = part + static_cast<int64_t>(m) * r + k;
                const int64_t step = static_cast<int64_t>(M) * r;
                float v = 0.0f;
                int q = 0;
                for (; q + 8 <= S; q += 8) {
                    float a[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) a[u] = __ldcg(pp + (q + u) * step);
#pragma unroll
                    for (int u = 0; u < 8; ++u) v += a[u];
                }
                for (; q < S; ++q) v += __ldcg(pp + q * step);
                t[static_cast<int64_t>(m) * r + k] = v;
            }
        }
        if (tid == 0) tickets[blockIdx.x] = 0u;  // restore for the next call
    }
}

constexpr int kS2Threads = 256;

template <int MB>
__global__ void __launch_bounds__(kS2Threads) decode_stage2_kernel(
    const uint32_t* __restrict__ U, int64_t ldu, const uint16_t* __restrict__ s1, const float* __restrict__ t,
    uint16_t* __restrict__ y, int M, int64_t d_out, int64_t r) {
    extern __shared__ float ts[];  // [MB][32][nw]: ts[(m*32 + c)*nw + w] = t[m][32w + c]
    const int nw = static_cast<int>(r / 32);
    const int tid = threadIdx.x;
    const int lane = tid & 31;

    pdl_wait();

    // consecutive threads fill consecutive words w of one (m, c) row: conflict-free stores
    for (int e = tid; e < MB * static_cast<int>(r); e += kS2Threads) {
        const int mc = e / nw;  // m * 32 + c
        const int w = e - mc * nw;
        const int m = mc >> 5;
        ts[e] = (m < M) ? t[static_cast<int64_t>(m) * r + 32 * w + (mc & 31)] : 0.0f;
    }
    __syncthreads();

    const int64_t warp = static_cast<int64_t>(blockIdx.x) * (kS2Threads / 32) + (tid >> 5);
    const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (kS2Threads / 32);
    for (int64_t i = warp; i < d_out; i += n_warps) {
        float acc[MB];
#pragma unroll
        for (int m = 0; m < MB; ++m) acc[m] = 0.0f;
        const uint32_t* urow = U + i * ldu;
        for (int w = lane; w < nw; w += 32) {
            const uint32_t nword = ~__ldg(urow + w);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const uint32_t flip = (nword << (31 - c)) & 0x80000000u;
#pragma unroll
                for (int m = 0; m < MB; ++m)
                    acc[m] += __uint_as_float(__float_as_uint(ts[(m * 32 + c) * nw + w]) ^ flip);
            }
        }
#pragma unroll
        for (int m = 0; m < MB; ++m) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
        }
        if (lane < M) {
            float v = acc[0];
#pragma unroll
            for (int m = 1; m < MB; ++m)
                if (lane == m) v = acc[m];
            y[static_cast<int64_t>(lane) * d_out + i] = float_to_bf16_bits(f16_bits_to_float(s1[i]) * v);
        }
    }
}

}  // namespace nq

// ------------------------------------------------------------------------------ host side
namespace {

struct DecodePlan {
    int64_t n_chunks;
    int S;
    int rows_per_slice;
    size_t off_t, off_part, off_tickets, total;
};

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
constexpr size_t kWsHeader = NQ_WS_HEADER_BYTES;

DecodePlan plan_decode(int64_t d_in, int64_t r, int64_t M) {
    DecodePlan p{};
    const int64_t nw = r / 32;
    p.n_chunks = (nw + nq::kS1WordsPerChunk - 1) / nq::kS1WordsPerChunk;
    const int64_t target = nq_host::sm_count();
    int64_t S = (target + p.n_chunks - 1) / p.n_chunks;
    if (S > 16) S = 16;                          // few partials: the last block sums them
    const int64_t min_s = (d_in + 2047) / 2048;  // at most 2048 rows per slice (z staging)
    if (S < min_s) S = min_s;
    if (S > d_in) S = d_in;
    if (S < 1) S = 1;
    p.rows_per_slice = static_cast<int>((d_in + S - 1) / S);
    p.S = static_cast<int>((d_in + p.rows_per_slice - 1) / p.rows_per_slice);
    // The tickets live at a fixed place, the first kWsHeader bytes of every workspace, so that
    // calls with different shapes (and the prefill path, which starts after the header too)
    // can share one workspace without landing data on a counter that must read zero.
    p.off_tickets = 0;
    p.off_t = kWsHeader;
    p.off_part = p.off_t + align256(static_cast<size_t>(M * r) * sizeof(float));
    p.total = p.off_part + align256(static_cast<size_t>(p.S) * M * r * sizeof(float));
    return p;
}

template <int MB>
nq_status launch_decode_mb(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int M, void* ws,
                           cudaStream_t stream, bool pdl) {
    const DecodePlan p = plan_decode(L->d_in, L->r, M);
    char* base = static_cast<char*>(ws);
    float* t = reinterpret_cast<float*>(base + p.off_t);
    float* part = reinterpret_cast<float*>(base + p.off_part);
    unsigned int* tickets = reinterpret_cast<unsigned int*>(base + p.off_tickets);

    using C = nq::S1Cfg<MB>;
    const size_t smem1 = (static_cast<size_t>(MB) * p.rows_per_slice + static_cast<size_t>(C::JG) * nq::pad32(C::OUT)) *
                         sizeof(float);
    static bool attr1 = false;
    if (!attr1) {
        cudaFuncSetAttribute(nq::decode_stage1_kernel<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        cudaFuncSetAttribute(nq::decode_stage2_kernel<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        attr1 = true;
    }
    {
        const uint32_t* V = L->V;
        int64_t ldv = L->ldv, d_in = L->d_in, r = L->r;
        const uint16_t* s2 = L->s2;
        int rps = p.rows_per_slice;
        void* args[] = {&V, &ldv, &s2, &x, &M, &d_in, &r, &rps, &part, &t, &tickets};
        dim3 grid(static_cast<unsigned>(p.n_chunks), static_cast<unsigned>(p.S));
        if (nq_host::launch_pdl(reinterpret_cast<const void*>(nq::decode_stage1_kernel<MB>), grid,
                                dim3(nq::kS1Threads), smem1, stream, args, pdl) != cudaSuccess)
            return NQ_ERR_LAUNCH;
    }
    {
        const uint32_t* U = L->U;
        int64_t ldu = L->ldu, d_out = L->d_out, r = L->r;
        const uint16_t* s1 = L->s1;
        const float* tc = t;
        void* args[] = {&U, &ldu, &s1, &tc, &y, &M, &d_out, &r};
        const size_t smem2 = static_cast<size_t>(MB) * L->r * sizeof(float);
        int64_t blocks = (L->d_out + 7) / 8;
        const int64_t cap = 2LL * nq_host::sm_count();
        if (blocks > cap) blocks = cap;
        if (nq_host::launch_pdl(reinterpret_cast<const void*>(nq::decode_stage2_kernel<MB>),
                                dim3(static_cast<unsigned>(blocks)), dim3(nq::kS2Threads), smem2, stream, args,
                                pdl) != cudaSuccess)
            return NQ_ERR_LAUNCH;
    }
    return NQ_OK;
}

}  // namespace

size_t nq_decode_workspace_bytes(int64_t d_in, int64_t r, int64_t M) { return plan_decode(d_in, r, M).total; }

// Shared-memory need of stage 2 (t staged per batch row): the caller rejects layers whose
// rank does not fit.
size_t nq_decode_stage2_smem(int64_t r, int64_t M) {
    const int64_t mb = M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8));
    return static_cast<size_t>(mb * r) * sizeof(float);
}

nq_status nq_launch_decode(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                           cudaStream_t stream, bool pdl) {
    const int m = static_cast<int>(M);
    if (M <= 1) return launch_decode_mb<1>(L, x, y, m, ws, stream, pdl);
    if (M <= 2) return launch_decode_mb<2>(L, x, y, m, ws, stream, pdl);
    if (M <= 4) return launch_decode_mb<4>(L, x, y, m, ws, stream, pdl);
    return launch_decode_mb<8>(L, x, y, m, ws, stream, pdl);
}
