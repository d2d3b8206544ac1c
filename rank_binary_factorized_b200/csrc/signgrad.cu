// signgrad.cu -- gradients with respect to the two sign factors.
//
// Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models"
// (research.samsung.com blog), section 3, "Step 3: Factorized Component Refinement": the latent
// factors are refined through sign() with straight-through estimators, so a training step needs
// dL/dU and dL/dV of the binary factors, which the identity estimator hands to the latents.
// For L = sum_m <ybar_m, y_m> and the section 2 equation read elementwise,
//
//   dL/dU_ik = s1_i sum_m ybar[m][i] T[m][k],   T = (x (.) s2) V        [M][r]
//   dL/dV_jk = s2_j sum_m x[m][j]    P[m][k],   P = (ybar (.) s1) U     [M][r]
//
// T is stage 1 of the forward; P is stage 1 of the exchanged layer (U <-> V, s1 <-> s2), i.e.
// of the transpose.  What remains is an outer-product sum over the M tokens with a dense fp32
// output of r (d_out + d_in) values:
//   M <= 8: T, P in fp32 from the decode stage 1; a CUDA-core kernel streams the output with
//           16-byte stores (HBM-write bound).
//   M > 8:  Z' = fp16(ybar (.) s1), P = fp16(Z' U) and Z = fp16(x (.) s2), T = fp16(Z V) from
//           the prefill GEMM 1; then dL/dU = Z'^T T and dL/dV = Z^T P on the tensor cores
//           (tcgen05, both operands MN-major by TMA, fp32 accumulators in TMEM, fp32 output by
//           TMA tile stores).  s1 and s2 ride in Z' and Z, as in the forward.
#include <algorithm>
#include <cstring>

#include "tc_common.cuh"

namespace nq {

// ------------------------------------------------------------------ M <= 8 (CUDA cores)
struct SignGradSmallArgs {
    const float* t;          // [M][r] fp32 (stage 1 of the layer)
    const float* p;          // [M][r] fp32 (stage 1 of the exchanged layer)
    const uint16_t* ybar;    // [M][d_out] bf16
    const uint16_t* x;       // [M][d_in] bf16
    const uint16_t* s1;      // [d_out] fp16
    const uint16_t* s2;      // [d_in] fp16
    float* gU;               // [d_out][ldgu]
    float* gV;               // [d_in][ldgv]
    int64_t ldgu, ldgv, d_out, d_in, r;
    int M;
    int rows_per_block;
};

// Row e of the concatenated row space: e < d_out is row e of dL/dU, otherwise row e - d_out of
// dL/dV.  A block owns 4 blockDim.x columns k (four per thread, one 16-byte store per row) and
// rows_per_block consecutive rows; T and P of its columns stay in registers.
template <int MM>
__global__ void __launch_bounds__(256) sign_grads_small_kernel(const SignGradSmallArgs a) {
    pdl_wait();
    const int64_t k = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    const bool kok = k < a.r;  // r % 32 == 0: a group of four is all in or all out
    float4 tv[MM], pv[MM];
#pragma unroll
    for (int m = 0; m < MM; ++m) {
        tv[m] = make_float4(0.f, 0.f, 0.f, 0.f);
        pv[m] = tv[m];
        if (m < a.M && kok) {
            tv[m] = *reinterpret_cast<const float4*>(a.t + m * a.r + k);
            pv[m] = *reinterpret_cast<const float4*>(a.p + m * a.r + k);
        }
    }
    const int64_t rows = a.d_out + a.d_in;
    const int64_t e0 = static_cast<int64_t>(blockIdx.y) * a.rows_per_block;
    const int64_t e1 = min(rows, e0 + a.rows_per_block);
    for (int64_t e = e0; e < e1; ++e) {
        const bool is_u = e < a.d_out;
        const int64_t row = is_u ? e : e - a.d_out;
        const int64_t n = is_u ? a.d_out : a.d_in;
        const uint16_t* act = (is_u ? a.ybar : a.x) + row;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < MM; ++m) {
            if (m < a.M) {
                const float c = bf16_bits_to_float(act[m * n]);
                const float4 v = is_u ? tv[m] : pv[m];
                acc.x = fmaf(c, v.x, acc.x);
                acc.y = fmaf(c, v.y, acc.y);
                acc.z = fmaf(c, v.z, acc.z);
                acc.w = fmaf(c, v.w, acc.w);
            }
        }
        const float sc = f16_bits_to_float(is_u ? a.s1[row] : a.s2[row]);
        acc.x *= sc;
        acc.y *= sc;
        acc.z *= sc;
        acc.w *= sc;
        if (kok) {
            float* dst = is_u ? a.gU + row * a.ldgu + k : a.gV + row * a.ldgv + k;
            __stcs(reinterpret_cast<float4*>(dst), acc);
        }
    }
}

// ------------------------------------------------------------------ M > 8 (tcgen05)
//
// D[w][n] = sum_m A[m][w] B[m][n]: A = Z' (or Z) [M][rows], B = T (or P) [M][r], both fp16 and
// stored with the token index m outermost, so both MMA operands are MN-major.  A stage holds
// 64 tokens: A as two TMA boxes of 64 rows-of-D x 64 tokens, B as tile_n / 64 boxes of 64
// rank columns x 64 tokens, each box 8 KB in the 128-byte swizzle (row = token, 128 bytes =
// 64 MN elements).  In the UMMA view a box is a column of 8-token swizzle atoms 1024 B apart
// (stride byte offset) and neighbouring boxes are the next 64 MN elements (leading byte
// offset 8192).
constexpr int kSgTileW = 128;    // MMA M: rows of the gradient per tile
constexpr int kSgTileK = 64;     // tokens per stage
constexpr int kSgBox = 8192;     // one 64 x 64 fp16 box
constexpr int kSgMaxStages = 8;
constexpr int kSgThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kSgStoreBox = 32 * 32 * 4;  // epilogue staging: 32 rows x 32 fp32 (128 B rows)
constexpr int kSgStoreBytes = 4 * 2 * kSgStoreBox;  // four warps, double-buffered
constexpr int kSgTmemCols = 512;

struct SignGradProblem {
    int64_t rows;       // d_out (dL/dU) or d_in (dL/dV)
    int n_tiles_w;      // row tiles
    int tile_begin;     // first global tile index of this problem
};

struct SignGradArgs {
    SignGradProblem pr[2];
    int n_tiles;        // both problems
    int n_tiles_n;      // rank tiles (same for both)
    int tile_n;         // rank columns per tile (multiple of 64, <= 256)
    int stages;
    int n_kblocks;      // ceil(M / 64)
    int64_t r;
    unsigned int* err;
};

__global__ void __launch_bounds__(kSgThreads, 1)
    sign_grads_umma_kernel(const __grid_constant__ CUtensorMap a0, const __grid_constant__ CUtensorMap b0,
                           const __grid_constant__ CUtensorMap d0, const __grid_constant__ CUtensorMap a1,
                           const __grid_constant__ CUtensorMap b1, const __grid_constant__ CUtensorMap d1,
                           const SignGradArgs args) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t smem_base = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
    const int tile_n = args.tile_n;
    const int nb = tile_n / 64;  // B boxes per stage
    const uint32_t stage_bytes = 2u * kSgBox + static_cast<uint32_t>(nb) * kSgBox;
    const int stages = args.stages;
    const uint32_t store_base = smem_base + stages * stage_bytes;
    const uint32_t bar_base = store_base + kSgStoreBytes;
    auto full = [&](int s) { return bar_base + 8u * s; };
    auto empty = [&](int s) { return bar_base + 8u * (kSgMaxStages + s); };
    auto acc_full = [&](int a) { return bar_base + 8u * (2 * kSgMaxStages + a); };
    auto acc_empty = [&](int a) { return bar_base + 8u * (2 * kSgMaxStages + 2 + a); };
    const uint32_t drain_bar = bar_base + 8u * (2 * kSgMaxStages + 4);
    const uint32_t tmem_slot = bar_base + 8u * (2 * kSgMaxStages + 5);
    auto a_tile = [&](int s) { return smem_base + s * stage_bytes; };
    auto b_tile = [&](int s) { return smem_base + s * stage_bytes + 2u * kSgBox; };
    // global tile -> (problem, row tile, rank tile); rank tiles vary fastest, so the CTAs of a
    // wave share their A tiles in L2
    auto locate = [&](int tile, int& pb, int& tw, int& tn) {
        pb = tile >= args.pr[1].tile_begin ? 1 : 0;
        const int local = tile - (pb ? args.pr[1].tile_begin : 0);
        tw = local / args.n_tiles_n;
        tn = local - tw * args.n_tiles_n;
    };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    unsigned int* err = args.err;
    const int n_tiles = args.n_tiles;
    const int nkb = args.n_kblocks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            tc::mbar_init(full(s), 1);
            tc::mbar_init(empty(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(acc_full(a), 1);
            tc::mbar_init(acc_empty(a), 4);
        }
        tc::mbar_init(drain_bar, 1);
        tc::mbar_fence_init();
        tc::tma_prefetch_desc(&a0);
        tc::tma_prefetch_desc(&b0);
        tc::tma_prefetch_desc(&a1);
        tc::tma_prefetch_desc(&b1);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, kSgTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem_raw + (tmem_slot - tc::smem_u32(smem_raw)));

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            pdl_wait();  // Z', T, Z, P are written by the grids queued before this one
            uint32_t it = 0, ph = 0;
            int s = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                int pb, tw, tn;
                locate(tile, pb, tw, tn);
                const CUtensorMap* ma = pb ? &a1 : &a0;
                const CUtensorMap* mb = pb ? &b1 : &b0;
                // boxes that lie wholly past the last row or rank column are not loaded: the
                // accumulator rows / columns they feed are never stored
                const int64_t arem = (pb ? args.pr[1].rows : args.pr[0].rows) - static_cast<int64_t>(tw) * kSgTileW;
                const int64_t brem = args.r - static_cast<int64_t>(tn) * tile_n;
                const int na = arem > 64 ? 2 : 1;
                const int nbv = static_cast<int>(min(static_cast<int64_t>(nb), (brem + 63) / 64));
                const uint32_t tx = static_cast<uint32_t>(na + nbv) * kSgBox;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    if (!(ok = tc::mbar_wait(empty(s), ph ^ 1u, err))) break;
                    tc::mbar_arrive_expect_tx(full(s), tx);
                    const int y = kb * kSgTileK;
                    for (int h = 0; h < na; ++h)
                        tc::tma_load_2d(a_tile(s) + h * kSgBox, ma, tw * kSgTileW + h * 64, y, full(s));
                    for (int h = 0; h < nbv; ++h)
                        tc::tma_load_2d(b_tile(s) + h * kSgBox, mb, tn * tile_n + h * 64, y, full(s));
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // drain: every load issued has landed before the CTA may exit
            const uint32_t first = it > static_cast<uint32_t>(stages) ? it - stages : 0u;
            for (uint32_t j = first; j < it; ++j) tc::mbar_wait(full(j % stages), (j / stages) & 1u, err);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_f16_f32(kSgTileW, tile_n, true, true);
            uint32_t tc_count = 0, ph = 0;
            int s = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++tc_count) {
                const int acc = tc_count & 1;
                const uint32_t aph = (tc_count >> 1) & 1u;
                if (!(ok = tc::mbar_wait(acc_empty(acc), aph ^ 1u, err))) break;
                tc::tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!(ok = tc::mbar_wait(full(s), ph, err))) break;
                    tc::tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kSgTileK / 16; ++kk) {
                        // 16 tokens = two 8-token atoms, 2048 B into every box
                        const uint64_t adesc = tc::smem_desc_sw128(a_tile(s) + kk * 2048u, kSgBox, 1024u);
                        const uint64_t bdesc = tc::smem_desc_sw128(b_tile(s) + kk * 2048u, kSgBox, 1024u);
                        tc::mma_f16_ss(d_tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(empty(s));
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                tc::mma_commit(acc_full(acc));
            }
            // every MMA issued by this thread has completed before TMEM is released
            tc::mma_commit(drain_bar);
            tc::mbar_wait(drain_bar, 0u, err);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        // warp q (of the TMEM lane quarter q = warp & 3) owns rows 32q .. 32q + 31 of a tile.
        // Each 32 x 32 fp32 block goes TMEM -> registers -> a swizzled staging box (row = lane,
        // 16-byte chunk c at c ^ (lane & 7): eight lanes hit eight bank groups) -> TMA store,
        // which clips rows and columns outside the gradient.
        pdl_wait();  // the gradient buffers may still be read by the grid queued before this one
        const int q = warp & 3;
        const uint32_t stage0 = store_base + static_cast<uint32_t>(q) * 2u * kSgStoreBox;
        uint32_t tc_count = 0, nstore = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++tc_count) {
            int pb, tw, tn;
            locate(tile, pb, tw, tn);
            const CUtensorMap* md = pb ? &d1 : &d0;
            const int acc = tc_count & 1;
            const uint32_t aph = (tc_count >> 1) & 1u;
            if (!(ok = tc::mbar_wait(acc_full(acc), aph, err))) break;
            tc::tc_fence_after();
            const int64_t row0 = static_cast<int64_t>(tw) * kSgTileW + q * 32;
            const bool rows_ok = row0 < (pb ? args.pr[1].rows : args.pr[0].rows);  // warp-uniform
            for (int c0 = 0; c0 < tile_n; c0 += 32) {
                const int64_t col0 = static_cast<int64_t>(tn) * tile_n + c0;
                if (!rows_ok || col0 >= args.r) break;  // warp-uniform: nothing left to store
                uint32_t v[32];
                tc::tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * 256 + c0, v);
                tc::tmem_wait_ld();
                const uint32_t buf = stage0 + (nstore & 1u) * kSgStoreBox;
                if (nstore >= 2) {
                    if (lane == 0) tc::bulk_wait_group_read<1>();  // the store that used buf is done reading
                    __syncwarp();
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t dst = buf + lane * 128u + ((static_cast<uint32_t>(j) ^ (lane & 7u)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[4 * j]), "r"(v[4 * j + 1]),
                                 "r"(v[4 * j + 2]), "r"(v[4 * j + 3])
                                 : "memory");
                }
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tc::tma_store_2d(md, buf, static_cast<int32_t>(col0), static_cast<int32_t>(row0));
                    tc::bulk_commit_group();
                }
                ++nstore;
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(acc_empty(acc));
        }
        if (lane == 0) tc::bulk_wait_group<0>();  // the stores have completed before the CTA exits
        __syncwarp();
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, kSgTmemCols);
    }
}

}  // namespace nq

// ------------------------------------------------------------------------------ host side
#include <atomic>

namespace {

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
constexpr size_t kSgSmemMax = 227 * 1024;

// 2-D fp16 [rows][cols] (row stride ld elements), boxes of 64 x 64, 128-byte swizzle.
bool tmap_f16_box64(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld) {
    auto enc = nq_host::tensor_map_encoder();
    if (!enc || (ld * 2) % 16 != 0 || (reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 [rows][cols] (row stride ld elements) for 32 x 32 tile stores, 128-byte swizzle.
bool tmap_f32_store(CUtensorMap* map, float* base, int64_t rows, int64_t cols, int64_t ld) {
    auto enc = nq_host::tensor_map_encoder();
    if (!enc || (ld * 4) % 16 != 0 || (reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 4)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t sg_smem_bytes(int tile_n, int stages) {
    const size_t stage = static_cast<size_t>(2 + tile_n / 64) * nq::kSgBox;
    return 1024 /* alignment slack */ + stages * stage + nq::kSgStoreBytes + 8 * (2 * nq::kSgMaxStages + 6) + 16;
}

template <int MM>
nq_status launch_small(const nq::SignGradSmallArgs& a, cudaStream_t stream, bool pdl) {
    const int64_t rows = a.d_out + a.d_in;
    const unsigned gx = static_cast<unsigned>((a.r / 4 + 255) / 256);
    const unsigned gy = static_cast<unsigned>((rows + a.rows_per_block - 1) / a.rows_per_block);
    nq::SignGradSmallArgs args = a;
    void* kargs[] = {&args};
    return nq_host::launch_pdl(reinterpret_cast<const void*>(nq::sign_grads_small_kernel<MM>), dim3(gx, gy), dim3(256),
                               0, stream, kargs, pdl) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_LAUNCH;
}

}  // namespace

size_t nq_sign_grads_ws(const nq_lrb_layer* L, const nq_lrb_layer* X, int64_t M) {
    if (M <= NQ_MATVEC_MAX_M)
        return NQ_WS_HEADER_BYTES + 2 * align256(static_cast<size_t>(M * L->r) * sizeof(float));
    size_t oz, ot, bl, bx;
    int64_t lz, lt;
    nq_prefill_stage1_layout(L, M, &oz, &lz, &ot, &lt, &bl);
    nq_prefill_stage1_layout(X, M, &oz, &lz, &ot, &lt, &bx);
    return align256(bl) + bx;
}

// L the layer, X its exchanged form (U <-> V, s1 <-> s2, d_out <-> d_in).
nq_status nq_launch_sign_grads(const nq_lrb_layer* L, const nq_lrb_layer* X, const uint16_t* x, const uint16_t* ybar,
                               int64_t M, float* gU, int64_t ldgu, float* gV, int64_t ldgv, void* ws,
                               cudaStream_t stream, bool pdl) {
    char* w = static_cast<char*>(ws);
    nq_status st;
    if (M <= NQ_MATVEC_MAX_M) {
        float* t = reinterpret_cast<float*>(w + NQ_WS_HEADER_BYTES);
        float* p = reinterpret_cast<float*>(w + NQ_WS_HEADER_BYTES + align256(static_cast<size_t>(M * L->r) * 4));
        if ((st = nq_launch_decode_stage1_pair(L, x, t, X, ybar, p, M, stream, pdl)) != NQ_OK) return st;
        nq::SignGradSmallArgs a{};
        a.t = t;
        a.p = p;
        a.ybar = ybar;
        a.x = x;
        a.s1 = L->s1;
        a.s2 = L->s2;
        a.gU = gU;
        a.gV = gV;
        a.ldgu = ldgu;
        a.ldgv = ldgv;
        a.d_out = L->d_out;
        a.d_in = L->d_in;
        a.r = L->r;
        a.M = static_cast<int>(M);
        // 16 rows per block, more when the grid would exceed its 65535 rows
        const int64_t rows = L->d_out + L->d_in;
        a.rows_per_block = static_cast<int>(std::max<int64_t>(16, (rows + 65534) / 65535));
        if (M <= 1) return launch_small<1>(a, stream, pdl);
        if (M <= 2) return launch_small<2>(a, stream, pdl);
        if (M <= 4) return launch_small<4>(a, stream, pdl);
        return launch_small<8>(a, stream, pdl);
    }

    // region of the layer's GEMM 1 (Z, T), then the exchanged layer's (Z', P)
    size_t oz, ot, bl, ozx, otx, bx;
    int64_t ldz, ldt, ldzx, ldtx;
    nq_prefill_stage1_layout(L, M, &oz, &ldz, &ot, &ldt, &bl);
    nq_prefill_stage1_layout(X, M, &ozx, &ldzx, &otx, &ldtx, &bx);
    char* wx = w + align256(bl);
    if ((st = nq_launch_prefill_stage1(L, x, M, w, stream, pdl)) != NQ_OK) return st;
    if ((st = nq_launch_prefill_stage1(X, ybar, M, wx, stream, pdl)) != NQ_OK) return st;
    const uint16_t* Z = reinterpret_cast<const uint16_t*>(w + oz);
    const uint16_t* T = reinterpret_cast<const uint16_t*>(w + ot);
    const uint16_t* Zx = reinterpret_cast<const uint16_t*>(wx + ozx);
    const uint16_t* P = reinterpret_cast<const uint16_t*>(wx + otx);

    // dL/dU = Z'^T T (rows d_out), dL/dV = Z^T P (rows d_in)
    CUtensorMap a0, b0, d0, a1, b1, d1;
    if (!tmap_f16_box64(&a0, Zx, M, L->d_out, ldzx) || !tmap_f16_box64(&b0, T, M, L->r, ldt) ||
        !tmap_f32_store(&d0, gU, L->d_out, L->r, ldgu) || !tmap_f16_box64(&a1, Z, M, L->d_in, ldz) ||
        !tmap_f16_box64(&b1, P, M, L->r, ldtx) || !tmap_f32_store(&d1, gV, L->d_in, L->r, ldgv))
        return NQ_ERR_LAUNCH;
    nq::SignGradArgs a{};
    a.tile_n = static_cast<int>(std::min<int64_t>(256, (L->r + 63) / 64 * 64));
    a.n_tiles_n = static_cast<int>((L->r + a.tile_n - 1) / a.tile_n);
    a.pr[0].rows = L->d_out;
    a.pr[0].n_tiles_w = static_cast<int>((L->d_out + nq::kSgTileW - 1) / nq::kSgTileW);
    a.pr[0].tile_begin = 0;
    a.pr[1].rows = L->d_in;
    a.pr[1].n_tiles_w = static_cast<int>((L->d_in + nq::kSgTileW - 1) / nq::kSgTileW);
    a.pr[1].tile_begin = a.pr[0].n_tiles_w * a.n_tiles_n;
    a.n_tiles = a.pr[1].tile_begin + a.pr[1].n_tiles_w * a.n_tiles_n;
    a.n_kblocks = static_cast<int>((M + nq::kSgTileK - 1) / nq::kSgTileK);
    a.r = L->r;
    a.err = nq_host::error_word();
    int stages = nq::kSgMaxStages;
    while (stages > 2 && sg_smem_bytes(a.tile_n, stages) > kSgSmemMax) --stages;
    a.stages = stages;
    const size_t smem = sg_smem_bytes(a.tile_n, stages);

    static std::atomic<bool> attr_done[64];  // per device; setting an attribute twice is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(nq::sign_grads_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kSgSmemMax)) != cudaSuccess)
            return NQ_ERR_LAUNCH;
        attr_done[dev].store(true, std::memory_order_release);
    }
    int grid = nq_host::sm_count();
    if (grid > a.n_tiles) grid = a.n_tiles;
    void* kargs[] = {&a0, &b0, &d0, &a1, &b1, &d1, &a};
    return nq_host::launch_pdl(reinterpret_cast<const void*>(nq::sign_grads_umma_kernel), dim3(grid),
                               dim3(nq::kSgThreads), smem, stream, kargs, pdl) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_LAUNCH;
}
