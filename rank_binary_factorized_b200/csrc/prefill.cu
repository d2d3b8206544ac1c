// prefill.cu -- M > 8 rows ("batch processing" GEMM of section 4, "Inference Performance",
// page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models",
// research.samsung.com blog) on the 5th-generation tensor cores.
//
// The factorisation equation of section 2 is evaluated right to left as two dense products
// whose weight operand is +-1:
//
//   Z = fp16(x (.) s2)                      [M][d_in]   (scale_convert_kernel)
//   T = fp16(Z V)        V in {+-1}^{d_in x r}          (umma kernel, mode V)
//   Y = bf16(s1 (.) (T U^T))  U in {+-1}^{d_out x r}    (umma kernel, mode U)
//
// Both products run in one persistent warp-specialised kernel, D[w][n] = sum_K A[w][K] B[n][K]:
//   * A (the weights, MMA M = 128 rows of U, or of V^T) is expanded on chip from the packed
//     words to fp16 +-1 by eight producer warps that write the UMMA 128-byte-swizzled
//     layout straight into shared memory (K-major for U, whose bits run along K = r;
//     MN-major for V^T, whose bits run along M = r);
//   * B (the activations Z or T, MMA N = up to 256 tokens) arrives by TMA tile loads;
//   * one thread issues tcgen05.mma (kind::f16, fp32 accumulate) into a double-buffered TMEM
//     accumulator, releasing smem stages with tcgen05.commit;
//   * four epilogue warps read TMEM (tcgen05.ld), apply s1 (mode U) and store.
// Every mbarrier wait is bounded in time; on expiry the kernel records a timeout in the
// error word, drains its own copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include "tc_common.cuh"

namespace nq {

constexpr int kTileW = 128;       // MMA M: weight rows per tile
constexpr int kTileK = 64;        // K per pipeline stage (one 128-byte swizzle row of fp16)
constexpr int kStages = 4;
constexpr int kTmemCols = 512;
constexpr int kExpandWarps = 8;     // warps 2..9 expand the packed weights
constexpr int kEpiWarp0 = 2 + kExpandWarps;  // warps 10..13: epilogue
constexpr int kPrefillThreads = 32 * (kEpiWarp0 + 4);
constexpr int kABytes = kTileW * kTileK * 2;  // 16 KB

enum PrefillMode : int { kModeV = 0, kModeU = 1 };

struct PrefillArgs {
    const uint32_t* bits;  // U [rows_w][ld] (mode U) or V [K][ld] (mode V)
    int64_t ld;            // words per row of `bits`
    int64_t rows_w;        // MMA-M extent: d_out (mode U) or r (mode V)
    int64_t K;             // reduction extent: r (mode U) or d_in (mode V)
    int64_t nwords;        // valid words per row of `bits` (r / 32)
    int64_t M;             // tokens
    int tile_n;            // tokens per tile (multiple of 16, <= 256)
    int n_tiles_w, n_tiles_n, n_kblocks;
    void* out;             // mode V: T fp16 [M][ldo]; mode U: Y bf16 [M][ldo]
    int64_t ldo;
    const uint16_t* s1;    // mode U
    unsigned int* err;
};

// fp16 +1 = 0x3C00, -1 = 0xBC00; two elements per 32-bit word, element 2i in the low half.
// Expands the 8 bits of `byte` (element e = bit e) into 8 fp16 values (16 bytes).
// `nbyte` holds the complemented bits (1 = negative) in its low 8 bits and zeros above.
// For pair q, (nbyte >> 2q) * 0x40008000 puts bit 2q at bit 15 and bit 2q+1 at bit 31: the
// product's two shifted copies occupy bits 15..22 and 30..31 (higher bits fall off), so they
// never overlap and no carry disturbs the two sign positions.
__device__ __forceinline__ uint4 expand_nbyte_pm1(uint32_t nbyte) {
    uint32_t r[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) r[q] = 0x3C003C00u | (((nbyte >> (2 * q)) * 0x40008000u) & 0x80008000u);
    return make_uint4(r[0], r[1], r[2], r[3]);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    lrb_umma_kernel(const __grid_constant__ CUtensorMap tmap_b, const PrefillArgs args) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base (the 128-byte swizzle pattern is a function of address bits 4-9)
    const uint32_t smem_base = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
    const int tile_n = args.tile_n;
    const uint32_t b_bytes = static_cast<uint32_t>(tile_n) * kTileK * 2;
    const uint32_t stage_bytes = kABytes + ((b_bytes + 1023u) & ~1023u);
    const uint32_t bar_base = smem_base + kStages * stage_bytes;
    // barriers: full_a[S], full_b[S], empty[S], acc_full[2], acc_empty[2], drain
    auto full_a = [&](int s) { return bar_base + 8u * s; };
    auto full_b = [&](int s) { return bar_base + 8u * (kStages + s); };
    auto empty = [&](int s) { return bar_base + 8u * (2 * kStages + s); };
    auto acc_full = [&](int a) { return bar_base + 8u * (3 * kStages + a); };
    auto acc_empty = [&](int a) { return bar_base + 8u * (3 * kStages + 2 + a); };
    const uint32_t drain_bar = bar_base + 8u * (3 * kStages + 4);
    const uint32_t tmem_slot = bar_base + 8u * (3 * kStages + 5);
    auto a_tile = [&](int s) { return smem_base + s * stage_bytes; };
    auto b_tile = [&](int s) { return smem_base + s * stage_bytes + kABytes; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(full_a(s), kExpandWarps);
            tc::mbar_init(full_b(s), 1);
            tc::mbar_init(empty(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(acc_full(a), 1);
            tc::mbar_init(acc_empty(a), 4);
        }
        tc::mbar_init(drain_bar, 1);
        tc::mbar_fence_init();
        tc::tma_prefetch_desc(&tmap_b);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem_raw + (tmem_slot - tc::smem_u32(smem_raw)));

    const int n_tiles = args.n_tiles_w * args.n_tiles_n;
    const int nkb = args.n_kblocks;
    unsigned int* err = args.err;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer (B)
        if (lane == 0) {
            pdl_wait();  // activations are written by the grid queued before this one
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                const int tn = tile / args.n_tiles_w;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!(ok = tc::mbar_wait(empty(s), ph ^ 1u, err))) break;
                    tc::mbar_arrive_expect_tx(full_b(s), b_bytes);
                    tc::tma_load_2d(b_tile(s), &tmap_b, kb * kTileK, tn * tile_n, full_b(s));
                }
            }
            // drain: every load issued has landed before the CTA may exit
            const uint32_t first = it > static_cast<uint32_t>(kStages) ? it - kStages : 0u;
            for (uint32_t j = first; j < it; ++j) tc::mbar_wait(full_b(j % kStages), (j / kStages) & 1u, err);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr bool a_mn = (MODE == kModeV);
            const uint32_t idesc = tc::idesc_f16_f32(kTileW, tile_n, a_mn, false);
            uint32_t it = 0, tc_count = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++tc_count) {
                const int acc = tc_count & 1;
                const uint32_t aph = (tc_count >> 1) & 1u;
                if (!(ok = tc::mbar_wait(acc_empty(acc), aph ^ 1u, err))) break;
                tc::tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!(ok = tc::mbar_wait(full_a(s), ph, err))) break;
                    if (!(ok = tc::mbar_wait(full_b(s), ph, err))) break;
                    tc::tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kTileK / 16; ++kk) {
                        uint64_t adesc;
                        if (MODE == kModeV) {
                            // MN-major: atoms of 64 (M) x 8 (K); M-groups 1024 B apart, K-groups 2048 B
                            adesc = tc::smem_desc_sw128(a_tile(s) + kk * 4096u, 1024u, 2048u);
                        } else {
                            // K-major: atoms of 8 rows x 64 K; 8-row groups 1024 B apart
                            adesc = tc::smem_desc_sw128(a_tile(s) + kk * 32u, 16u, 1024u);
                        }
                        const uint64_t bdesc = tc::smem_desc_sw128(b_tile(s) + kk * 32u, 16u, 1024u);
                        tc::mma_f16_ss(d_tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(empty(s));
                }
                if (!ok) break;
                tc::mma_commit(acc_full(acc));
            }
            // every MMA issued by this thread has completed before TMEM is released
            tc::mma_commit(drain_bar);
            tc::mbar_wait(drain_bar, 0u, err);
        }
    } else if (warp < kEpiWarp0) {
        // ---------------------------------------------------------------- A expansion (weights)
        // 256 threads, one packed word (32 weights) per thread per k block:
        //  U (K-major): row = t / 2, word 2 kb + (t & 1) -> chunks 4 (t & 1) .. +3 of the row
        //  V (MN-major): K-row jl, M-group h, word `half` of that group; lanes 0..7 of every
        //  8-lane group take eight different K-rows so their 16-byte stores hit distinct banks
        const int t = threadIdx.x - 64;  // 0..255
        // Each thread's packed word is loaded kPrefetch iterations ahead of its use into a
        // register ring, so the L2/DRAM latency of the words overlaps the expansion and the
        // waits of the iterations before.  The load address comes from per-thread constants
        // and a (tile, k block) cursor that only ever increments (no integer division).
        int64_t row_off;  // row index within a tile (U) or within a k block (V)
        int word_off;     // word offset within the k block (U) or within the tile's 4 words (V)
        if (MODE == kModeU) {
            row_off = t >> 1;
            word_off = t & 1;
        } else {
            row_off = (t & 7) | ((t >> 5) << 3);
            word_off = ((t >> 4) & 1) * 2 + ((t >> 3) & 1);
        }
        int pf_tile = blockIdx.x, pf_kb = 0, pf_tw = blockIdx.x % args.n_tiles_w;
        auto load_next = [&](uint32_t& w) {
            w = 0u;
            if (pf_tile < n_tiles) {
                int64_t row, wcol;
                bool row_ok;
                if (MODE == kModeU) {
                    row = static_cast<int64_t>(pf_tw) * kTileW + row_off;
                    wcol = static_cast<int64_t>(pf_kb) * 2 + word_off;
                    row_ok = row < args.rows_w;
                } else {
                    row = static_cast<int64_t>(pf_kb) * kTileK + row_off;
                    wcol = static_cast<int64_t>(pf_tw) * (kTileW / 32) + word_off;
                    row_ok = row < args.K;
                }
                if (row_ok && wcol < args.nwords) w = __ldg(args.bits + row * args.ld + wcol);
                if (++pf_kb == nkb) {
                    pf_kb = 0;
                    pf_tile += gridDim.x;
                    pf_tw += gridDim.x;
                    while (pf_tw >= args.n_tiles_w) pf_tw -= args.n_tiles_w;
                }
            }
        };
        constexpr int kPrefetch = 4;
        uint32_t ring[kPrefetch];
#pragma unroll
        for (int i = 0; i < kPrefetch; ++i) load_next(ring[i]);
        const int my_tiles = (n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
        const uint32_t total_it = static_cast<uint32_t>(my_tiles > 0 ? my_tiles : 0) * static_cast<uint32_t>(nkb);
        bool ok = true;
        for (uint32_t it = 0; it < total_it && ok; ++it) {
            const int s = it % kStages;
            const uint32_t ph = (it / kStages) & 1u;
            const uint32_t wcur = ring[0];
#pragma unroll
            for (int i = 0; i + 1 < kPrefetch; ++i) ring[i] = ring[i + 1];
            load_next(ring[kPrefetch - 1]);
            if (!(ok = tc::mbar_wait(empty(s), ph ^ 1u, err))) break;
            const uint32_t a = a_tile(s);
            const uint32_t nw = ~wcur;
            if (MODE == kModeU) {
                // half (t & 1) of row t/2 of a K-major SW128 tile: chunks 4 (t & 1) .. +3
                const int row = t >> 1, c0 = 4 * (t & 1);
                const uint32_t row_base = a + (row >> 3) * 1024u + (row & 7) * 128u;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    sts128(row_base + (((c0 + c) ^ (row & 7)) << 4), expand_nbyte_pm1((nw >> (8 * c)) & 0xFFu));
            } else {
                const int jl = (t & 7) | ((t >> 5) << 3), half = (t >> 3) & 1, h = (t >> 4) & 1;
                const uint32_t atom = a + ((jl >> 3) * 2 + h) * 1024u + (jl & 7) * 128u;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    sts128(atom + (((4 * half + c) ^ (jl & 7)) << 4), expand_nbyte_pm1((nw >> (8 * c)) & 0xFFu));
            }
            // each lane makes its own stores visible to the tensor core's (async) proxy; one
            // arrive per warp after the warp has converged
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(full_a(s));
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        pdl_wait();  // the outputs may still be read by the grid queued before this one
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int rl = q * 32 + lane;  // accumulator row (TMEM lane)
        uint32_t tc_count = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++tc_count) {
            const int tw = tile % args.n_tiles_w;
            const int tn = tile / args.n_tiles_w;
            const int acc = tc_count & 1;
            const uint32_t aph = (tc_count >> 1) & 1u;
            if (!(ok = tc::mbar_wait(acc_full(acc), aph, err))) break;
            tc::tc_fence_after();
            const int64_t wrow = static_cast<int64_t>(tw) * kTileW + rl;
            const bool row_ok = wrow < args.rows_w;
            float scale = 1.0f;
            if (MODE == kModeU && row_ok) scale = f16_bits_to_float(args.s1[wrow]);
            for (int c0 = 0; c0 < tile_n; c0 += 32) {
                uint32_t v[32];
                tc::tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * 256 + c0, v);
                tc::tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int64_t tok = static_cast<int64_t>(tn) * tile_n + c0 + j;
                        if (c0 + j < tile_n && tok < args.M) {
                            const float f = __uint_as_float(v[j]);
                            if (MODE == kModeU) {
                                static_cast<uint16_t*>(args.out)[tok * args.ldo + wrow] = float_to_bf16_bits(scale * f);
                            } else {
                                static_cast<uint16_t*>(args.out)[tok * args.ldo + wrow] =
                                    __half_as_ushort(__float2half_rn(f));
                            }
                        }
                    }
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(acc_empty(acc));
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Z[m][j] = fp16(bf16 x[m][j] * fp16 s2[j]) for j < d_in; row stride ldz.
__global__ void __launch_bounds__(256) scale_convert_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ s2,
                                                           uint16_t* __restrict__ z, int64_t M, int64_t d_in, int64_t ldz) {
    pdl_wait();
    const int64_t total = M * d_in;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = e / d_in;
        const int64_t j = e - m * d_in;
        const float v = bf16_bits_to_float(x[e]) * f16_bits_to_float(s2[j]);
        z[m * ldz + j] = __half_as_ushort(__float2half_rn(v));
    }
}

}  // namespace nq

// ------------------------------------------------------------------------------ host side
namespace {

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

struct PrefillPlan {
    int64_t ldz, ldt;
    size_t off_z, off_t, total;
};

PrefillPlan plan_prefill(const nq_lrb_layer* L, int64_t M) {
    PrefillPlan p{};
    p.ldz = round_up(L->d_in, 8);  // 16-byte aligned rows for TMA
    p.ldt = round_up(L->r, 8);
    p.off_z = NQ_WS_HEADER_BYTES;  // the header belongs to the decode path's tickets
    p.off_t = p.off_z + align256(static_cast<size_t>(M * p.ldz) * 2);
    p.total = p.off_t + align256(static_cast<size_t>(M * p.ldt) * 2);
    return p;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// 2-D fp16 tensor [rows][cols] with row stride ld elements; box = 64 (inner) x box_rows.
bool make_tmap(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(nq::kTileK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t umma_smem_bytes(int tile_n) {
    const size_t b = static_cast<size_t>(tile_n) * nq::kTileK * 2;
    const size_t stage = nq::kABytes + ((b + 1023) & ~static_cast<size_t>(1023));
    return 1024 /* alignment slack */ + nq::kStages * stage + 8 * (3 * nq::kStages + 6) + 16;
}

template <int MODE>
nq_status launch_umma(const nq::PrefillArgs& a, const CUtensorMap& map, cudaStream_t stream, bool pdl) {
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const size_t smem = umma_smem_bytes(256);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(nq::lrb_umma_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return NQ_ERR_LAUNCH;
        attr_done[dev] = true;
    }
    const int tiles = a.n_tiles_w * a.n_tiles_n;
    int grid = nq_host::sm_count();
    if (grid > tiles) grid = tiles;
    nq::PrefillArgs args = a;
    CUtensorMap tm = map;
    void* kargs[] = {&tm, &args};
    return nq_host::launch_pdl(reinterpret_cast<const void*>(nq::lrb_umma_kernel<MODE>), dim3(grid),
                               dim3(nq::kPrefillThreads), umma_smem_bytes(a.tile_n), stream, kargs, pdl) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_LAUNCH;
}

}  // namespace

size_t nq_prefill_workspace_bytes(const nq_lrb_layer* L, int64_t M) { return plan_prefill(L, M).total; }

nq_status nq_launch_prefill(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                            cudaStream_t stream, bool pdl) {
    const PrefillPlan p = plan_prefill(L, M);
    uint16_t* z = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + p.off_z);
    uint16_t* t = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + p.off_t);
    unsigned int* err = nq_host::error_word();
    const int tile_n = M >= 256 ? 256 : static_cast<int>(round_up(M, 16));

    {  // Z = fp16(x * s2)
        int64_t blocks = (M * L->d_in + 255) / 256;
        const int64_t cap = 4LL * nq_host::sm_count();
        if (blocks > cap) blocks = cap;
        const uint16_t* s2 = L->s2;
        int64_t d_in = L->d_in, ldz = p.ldz;
        void* args[] = {&x, &s2, &z, &M, &d_in, &ldz};
        if (nq_host::launch_pdl(reinterpret_cast<const void*>(nq::scale_convert_kernel), dim3(static_cast<unsigned>(blocks)),
                                dim3(256), 0, stream, args, pdl) != cudaSuccess)
            return NQ_ERR_LAUNCH;
    }
    {  // T = fp16(Z V): weights = V^T (M-extent r, K = d_in), B = Z
        CUtensorMap map;
        if (!make_tmap(&map, z, M, L->d_in, p.ldz, tile_n)) return NQ_ERR_LAUNCH;
        nq::PrefillArgs a{};
        a.bits = L->V;
        a.ld = L->ldv;
        a.rows_w = L->r;
        a.K = L->d_in;
        a.nwords = L->r / 32;
        a.M = M;
        a.tile_n = tile_n;
        a.n_tiles_w = static_cast<int>((L->r + nq::kTileW - 1) / nq::kTileW);
        a.n_tiles_n = static_cast<int>((M + tile_n - 1) / tile_n);
        a.n_kblocks = static_cast<int>((L->d_in + nq::kTileK - 1) / nq::kTileK);
        a.out = t;
        a.ldo = p.ldt;
        a.s1 = nullptr;
        a.err = err;
        nq_status st = launch_umma<nq::kModeV>(a, map, stream, pdl);
        if (st != NQ_OK) return st;
    }
    {  // Y = bf16(s1 * (T U^T)): weights = U (M-extent d_out, K = r), B = T
        CUtensorMap map;
        if (!make_tmap(&map, t, M, L->r, p.ldt, tile_n)) return NQ_ERR_LAUNCH;
        nq::PrefillArgs a{};
        a.bits = L->U;
        a.ld = L->ldu;
        a.rows_w = L->d_out;
        a.K = L->r;
        a.nwords = L->r / 32;
        a.M = M;
        a.tile_n = tile_n;
        a.n_tiles_w = static_cast<int>((L->d_out + nq::kTileW - 1) / nq::kTileW);
        a.n_tiles_n = static_cast<int>((M + tile_n - 1) / tile_n);
        a.n_kblocks = static_cast<int>((L->r + nq::kTileK - 1) / nq::kTileK);
        a.out = y;
        a.ldo = L->d_out;
        a.s1 = L->s1;
        a.err = err;
        nq_status st = launch_umma<nq::kModeU>(a, map, stream, pdl);
        if (st != NQ_OK) return st;
    }
    return NQ_OK;
}
