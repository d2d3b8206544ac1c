// prefill.cu -- M > 8 rows ("batch processing" GEMM of section 4, "Inference Performance",
// page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models",
// research.samsung.com blog) on the 5th-generation tensor cores.
//
// The factorisation equation of section 2 is evaluated right to left as two dense products
// whose weight operand is +-1:
//
//   Z = fp16(2^-e x (.) s2)                 [M][d_in]   (scale_convert_rows_kernel)
//   T = fp16(Z V)        V in {+-1}^{d_in x r}          (umma kernel, mode V)
//   Y = bf16(2^e s1 (.) (T U^T))  U in {+-1}^{d_out x r} (umma kernel, mode U)
// with one power of two e per token that keeps Z and T inside fp16's range (the sign-gradient
// path, which sums over tokens, uses e = 0: scale_convert_kernel).
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

#include <algorithm>
#include <cstring>

#include "tc_common.cuh"

namespace nq {

constexpr int kTileW = 128;       // MMA M: weight rows per tile
constexpr int kTileK = 64;        // K per pipeline stage (one 128-byte swizzle row of fp16)
constexpr int kMaxStages = 12;   // pipeline depth: as many stages as fit (fewer for wide tiles)
constexpr int kTmemCols = 512;
constexpr int kExpandWarps = 8;     // warps 2..9 expand the packed weights
constexpr int kExpandGroups = 2;    // in groups that fill alternate stages
constexpr int kGroupWarps = kExpandWarps / kExpandGroups;
static_assert(2 * 32 * kGroupWarps == 256, "a stage is 256 packed words, two per producer thread");
constexpr int kEpiWarp0 = 2 + kExpandWarps;  // warps 10..13: epilogue
constexpr int kPrefillThreads = 32 * (kEpiWarp0 + 4);
constexpr int kABytes = kTileW * kTileK * 2;  // 16 KB
// Packed-sign box a stage receives by TMA (4 words x 128 rows of U, or 4 words x 64 rows of V)
constexpr int kBitsWords = 4;
constexpr int kBitsBytes = kBitsWords * 4 * kTileW;  // slot size (2 KB)

enum PrefillMode : int { kModeV = 0, kModeU = 1 };

struct PrefillArgs {
    const uint32_t* bits;  // U [rows_w][ld] (mode U) or V [K][ld] (mode V)
    int64_t ld;            // words per row of `bits`
    int64_t rows_w;        // MMA-M extent: d_out (mode U) or r (mode V)
    int64_t K;             // reduction extent: r (mode U) or d_in (mode V)
    int64_t nwords;        // valid words per row of `bits` (r / 32)
    int64_t M;             // tokens
    int tile_n;            // tokens per tile (multiple of 16, <= 256)
    int stages;            // pipeline stages in shared memory (2 .. kMaxStages)
    int n_tiles_w, n_tiles_n, n_kblocks;
    void* out;             // mode V: T fp16 [M][ldo]; mode U: Y bf16 [M][ldo]
    int64_t ldo;
    const uint16_t* s1;    // mode U
    const int* row_exp;    // mode U: token m's activations were scaled by 2^-row_exp[m] (none if null)
    unsigned int* err;
    int bits_tma;          // packed signs arrive by TMA (row stride a multiple of 16 bytes)
    // gradient mode (mode U, gpart != nullptr): no Y; for every token tile tn and row w,
    // gpart[tn][w] = sum over the tile's tokens of cot[tok][w] * (T U^T)[tok][w] (fp64)
    const uint16_t* cot;   // [M][ldcot] bf16
    int64_t ldcot;
    double* gpart;         // [n_tiles_n][rows_w]
    // split over K (mode V with bits_tma only): every tile's k blocks are divided among ksplit
    // work units, each writing its fp32 partial product to partial[split][M][ldo]; a reduction
    // kernel then adds the splits in order and rounds to fp16
    int ksplit;
    float* partial;
};

// fp16 +1 = 0x3C00, -1 = 0xBC00; two elements per 32-bit word, element 2i in the low half.
// Expands the 8 bits of `byte` (element e = bit e, 1 = +1) into 8 fp16 values (16 bytes).
// For pair q, byte * (2^(15 - 2q) + 2^(30 - 2q)) puts bit 2q at bit 15 and bit 2q+1 at bit 31;
// the product's two shifted copies of the byte (bits 15-2q .. 22-2q and 30-2q .. 37-2q)
// never overlap, so no carry disturbs the two sign positions.  Masked, they are the signs of
// the two elements with 1 = +1; XOR with the pattern of (-1, -1) flips them into fp16 signs.
__device__ __forceinline__ uint4 expand_byte_pm1(uint32_t byte) {
    uint32_t r[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) r[q] = ((byte * (0x40008000u >> (2 * q))) & 0x80008000u) ^ 0xBC00BC00u;
    return make_uint4(r[0], r[1], r[2], r[3]);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// One 32-token chunk of GEMM 2's epilogue when some token carries a power of two (rare: rows
// outside fp16's range): the chunk is read from TMEM again and token j's values are multiplied
// by 2^e_j, e_j handed across the warp from lane j.  Kept out of line so that the plain loop
// stays compact.  Returns the chunk's share of the gradient partial (gradient mode).
__device__ __noinline__ double scaled_chunk(const PrefillArgs& args, uint32_t taddr, int tn, int tile_n, int c0,
                                            int64_t wrow, bool row_ok, float scale, bool grad, int el) {
    uint32_t v[32];
    tc::tmem_ld_32x32b_x32(taddr, v);
    tc::tmem_wait_ld();
    double g = 0.0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int e = __shfl_sync(__activemask(), el, j);
        const int64_t tok = static_cast<int64_t>(tn) * tile_n + c0 + j;
        if (row_ok && c0 + j < tile_n && tok < args.M) {
            const float f = __uint_as_float(v[j]);
            if (grad) {
                g += static_cast<double>(bf16_bits_to_float(args.cot[tok * args.ldcot + wrow])) *
                     (static_cast<double>(f) * __longlong_as_double(static_cast<long long>(1023 + e) << 52));
            } else {
                const float sf = scale * f;
                const float o = (e >= -126 && e <= 127) ? sf * __int_as_float((e + 127) << 23) : ldexpf(sf, e);
                static_cast<uint16_t*>(args.out)[tok * args.ldo + wrow] = float_to_bf16_bits(o);
            }
        }
    }
    return g;
}

// SPLIT: the launch splits tiles over K (mode V); without it the unit of work is the tile and
// the unit bookkeeping folds away at compile time.
template <int MODE, bool SPLIT>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    lrb_umma_kernel(const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_bits,
                    const PrefillArgs args) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base (the 128-byte swizzle pattern is a function of address bits 4-9)
    const uint32_t smem_base = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
    const int tile_n = args.tile_n;
    const uint32_t b_bytes = static_cast<uint32_t>(tile_n) * kTileK * 2;
    const uint32_t stage_bytes = kABytes + ((b_bytes + 1023u) & ~1023u) + kBitsBytes;
    const int stages = args.stages;
    const uint32_t bar_base = smem_base + stages * stage_bytes;
    // barriers: full_a[S], full_b[S], empty[S], acc_full[2], acc_empty[2], drain
    auto full_a = [&](int s) { return bar_base + 8u * s; };
    auto full_b = [&](int s) { return bar_base + 8u * (kMaxStages + s); };
    auto empty = [&](int s) { return bar_base + 8u * (2 * kMaxStages + s); };
    auto acc_full = [&](int a) { return bar_base + 8u * (3 * kMaxStages + a); };
    auto acc_empty = [&](int a) { return bar_base + 8u * (3 * kMaxStages + 2 + a); };
    const uint32_t drain_bar = bar_base + 8u * (3 * kMaxStages + 4);
    const uint32_t tmem_slot = bar_base + 8u * (3 * kMaxStages + 5);
    auto a_tile = [&](int s) { return smem_base + s * stage_bytes; };
    auto b_tile = [&](int s) { return smem_base + s * stage_bytes + kABytes; };
    auto bits_tile = [&](int s) { return smem_base + (s + 1) * stage_bytes - kBitsBytes; };
    // bytes of packed signs per stage and their box origin for k block kb of weight tile tw
    const uint32_t bits_bytes = (MODE == kModeU) ? kBitsWords * 4 * kTileW : kBitsWords * 4 * kTileK;
    auto bits_x = [&](int tw, int kb) { return (MODE == kModeU) ? (kb >> 1) * kBitsWords : tw * kBitsWords; };
    auto bits_y = [&](int tw, int kb) { return (MODE == kModeU) ? tw * kTileW : kb * kTileK; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            tc::mbar_init(full_a(s), kGroupWarps);
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
        if (args.bits_tma) tc::tma_prefetch_desc(&tmap_bits);
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
    // work unit u: tile u / ksplit, k blocks [kb_lo, kb_hi) of split u % ksplit
    const int ksplit = (MODE == kModeV && SPLIT) ? args.ksplit : 1;
    const int n_units = n_tiles * ksplit;
    auto unit_kb = [&](int u, int& kb_lo, int& kb_hi) {
        const int sp = u % ksplit;
        kb_lo = sp * nkb / ksplit;
        kb_hi = (sp + 1) * nkb / ksplit;
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer (B)
        if (lane == 0) {
            // the packed signs of the first `stages` k blocks are weights: load them before
            // waiting for the activations (the stage's barrier also waits for its B tile)
            uint32_t pre = 0;
            if (args.bits_tma) {
                int u = blockIdx.x, kb = 0, kb_lo = 0, kb_hi = nkb;
                if (u < n_units) unit_kb(u, kb_lo, kb_hi);
                kb = kb_lo;
                while (u < n_units && pre < static_cast<uint32_t>(stages)) {
                    const int tw = (u / ksplit) % args.n_tiles_w;
                    tc::mbar_expect_tx(full_b(pre), bits_bytes);
                    tc::tma_load_2d(bits_tile(pre), &tmap_bits, bits_x(tw, kb), bits_y(tw, kb), full_b(pre));
                    ++pre;
                    if (++kb == kb_hi) {
                        u += gridDim.x;
                        if (u < n_units) unit_kb(u, kb_lo, kb_hi);
                        kb = kb_lo;
                    }
                }
            }
            pdl_wait();  // activations are written by the grid queued before this one
            uint32_t it = 0, ph = 0;
            int s = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                const int tile = u / ksplit;
                const int tn = tile / args.n_tiles_w;
                const int tw = tile - tn * args.n_tiles_w;
                int kb_lo, kb_hi;
                unit_kb(u, kb_lo, kb_hi);
                for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
                    if (!(ok = tc::mbar_wait(empty(s), ph ^ 1u, err))) break;
                    if (args.bits_tma && it >= pre) {
                        tc::mbar_expect_tx(full_b(s), bits_bytes);
                        tc::tma_load_2d(bits_tile(s), &tmap_bits, bits_x(tw, kb), bits_y(tw, kb), full_b(s));
                    }
                    tc::mbar_arrive_expect_tx(full_b(s), b_bytes);
                    tc::tma_load_2d(b_tile(s), &tmap_b, kb * kTileK, tn * tile_n, full_b(s));
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // drain: every load issued has landed before the CTA may exit
            const uint32_t first = it > static_cast<uint32_t>(stages) ? it - stages : 0u;
            for (uint32_t j = first; j < it; ++j) tc::mbar_wait(full_b(j % stages), (j / stages) & 1u, err);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr bool a_mn = (MODE == kModeV);
            const uint32_t idesc = tc::idesc_f16_f32(kTileW, tile_n, a_mn, false);
            uint32_t tc_count = 0, ph = 0;
            int s = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++tc_count) {
                const int acc = tc_count & 1;
                const uint32_t aph = (tc_count >> 1) & 1u;
                if (!(ok = tc::mbar_wait(acc_empty(acc), aph ^ 1u, err))) break;
                tc::tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
                int kb_lo, kb_hi;
                unit_kb(u, kb_lo, kb_hi);
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
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
                        tc::mma_f16_ss(d_tmem, adesc, bdesc, idesc, (kb > kb_lo || kk > 0) ? 1u : 0u);
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
    } else if (warp < kEpiWarp0) {
        // ---------------------------------------------------------------- A expansion (weights)
        // kExpandGroups groups of warps take alternate k blocks, so that as many stages are
        // filled at once (a stage's stores, proxy fence and arrival are a latency chain).  A
        // stage holds 256 packed words; thread tg of a group owns two adjacent ones:
        //  U (K-major): row tg of the tile, words 2 kb and 2 kb + 1: the row's 64 K values, all
        //  eight 16-byte chunks of its 128-byte swizzled row
        //  V (MN-major): K-row jl = (tg & 7) | ((tg >> 4) << 3) of the k block, M-group
        //  h = (tg >> 3) & 1, words 2h and 2h + 1 of the tile's four (128 M values)
        // Lanes 0..7 of every 8-lane group take eight different rows, so their 16-byte stores
        // fall in eight different bank groups.
        const int grp = (warp - 2) / kGroupWarps;
        const int tg = threadIdx.x - 64 - grp * 32 * kGroupWarps;  // 0..127
        const int jl = (tg & 7) | ((tg >> 4) << 3), hgrp = (tg >> 3) & 1;
        const bool ld_even = (args.ld & 1) == 0;  // 8-byte loads of a word pair are aligned
        // The pair is loaded kPrefetch of the group's iterations ahead of its use into a
        // register ring, so the L2/DRAM latency overlaps the expansion and the waits of the
        // iterations before.  The (tile, k block) cursor only ever increments.
        int pf_tile = blockIdx.x, pf_kb = 0, pf_tw = blockIdx.x % args.n_tiles_w;
        auto advance = [&]() {
            if (++pf_kb == nkb) {
                pf_kb = 0;
                pf_tile += gridDim.x;
                pf_tw += gridDim.x;
                while (pf_tw >= args.n_tiles_w) pf_tw -= args.n_tiles_w;
            }
        };
        for (int i = 0; i < grp; ++i) advance();
        auto load_next = [&](uint2& w) {
            w = make_uint2(0u, 0u);
            if (pf_tile < n_tiles) {
                int64_t row, wcol;
                bool row_ok;
                if (MODE == kModeU) {
                    row = static_cast<int64_t>(pf_tw) * kTileW + tg;
                    wcol = 2 * static_cast<int64_t>(pf_kb);
                    row_ok = row < args.rows_w;
                } else {
                    row = static_cast<int64_t>(pf_kb) * kTileK + jl;
                    wcol = static_cast<int64_t>(pf_tw) * (kTileW / 32) + 2 * hgrp;
                    row_ok = row < args.K;
                }
                const uint32_t* src = args.bits + row * args.ld + wcol;
                if (row_ok) {
                    if (wcol + 1 < args.nwords) {
                        if (ld_even) {
                            w = __ldg(reinterpret_cast<const uint2*>(src));
                        } else {
                            w.x = __ldg(src);
                            w.y = __ldg(src + 1);
                        }
                    } else if (wcol < args.nwords) {
                        w.x = __ldg(src);
                    }
                }
            }
            for (int g = 0; g < kExpandGroups && pf_tile < n_tiles; ++g) advance();
        };
        constexpr int kPrefetch = 8;
        uint2 ring[kPrefetch];
        const int my_tiles = (n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
        uint32_t total_it = static_cast<uint32_t>(my_tiles > 0 ? my_tiles : 0) * static_cast<uint32_t>(nkb);
        if (ksplit > 1) {  // the k blocks of this CTA's work units
            total_it = 0;
            for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
                int kb_lo, kb_hi;
                unit_kb(u, kb_lo, kb_hi);
                total_it += static_cast<uint32_t>(kb_hi - kb_lo);
            }
        }
        // this thread's 128-byte smem row within a stage's A tile, and its swizzle
        const uint32_t row_off_b = (MODE == kModeU) ? (tg >> 3) * 1024u + (tg & 7) * 128u
                                                    : ((jl >> 3) * 2 + hgrp) * 1024u + (jl & 7) * 128u;
        const int swz = (MODE == kModeU) ? (tg & 7) : (jl & 7);
        // expands this thread's word pair into its 128-byte row of stage s's A tile and
        // publishes it to the tensor core's (async) proxy
        auto expand_store = [&](uint2 wcur, int s) {
            const uint32_t row_addr = a_tile(s) + row_off_b;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t byte = ((c < 4 ? wcur.x : wcur.y) >> (8 * (c & 3))) & 0xFFu;
                sts128(row_addr + ((c ^ swz) << 4), expand_byte_pm1(byte));
            }
            tc::fence_proxy_async_smem();
            __syncwarp();  // one arrive per warp after the warp has converged
            if (lane == 0) tc::mbar_arrive(full_a(s));
        };
        bool ok = true;
        int s = grp;  // stage and phase of iteration `it` (grp < 2 <= stages)
        uint32_t ph = 0;
        if (args.bits_tma) {
            // the stage's packed signs land with its B tile: wait for the stage, read them
            // from shared memory (rows of 16 bytes: 4 words)
            int cur_kb = grp % nkb;
            for (uint32_t it = grp; it < total_it && ok; it += kExpandGroups) {
                if (!(ok = tc::mbar_wait(full_b(s), ph, err))) break;
                const uint32_t src = bits_tile(s) + ((MODE == kModeU) ? tg * 16u + 8u * (cur_kb & 1) : jl * 16u + 8u * hgrp);
                uint2 w;
                asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w.x), "=r"(w.y) : "r"(src));
                expand_store(w, s);
                s += kExpandGroups;
                while (s >= stages) {
                    s -= stages;
                    ph ^= 1u;
                }
                cur_kb += kExpandGroups;
                while (cur_kb >= nkb) cur_kb -= nkb;
            }
        } else {
#pragma unroll
            for (int i = 0; i < kPrefetch; ++i) load_next(ring[i]);
            for (uint32_t it = grp; it < total_it && ok; it += kExpandGroups) {
                const uint2 wcur = ring[0];
#pragma unroll
                for (int j = 0; j + 1 < kPrefetch; ++j) ring[j] = ring[j + 1];
                load_next(ring[kPrefetch - 1]);
                if (!(ok = tc::mbar_wait(empty(s), ph ^ 1u, err))) break;
                expand_store(wcur, s);
                s += kExpandGroups;
                while (s >= stages) {
                    s -= stages;
                    ph ^= 1u;
                }
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        pdl_wait();  // the outputs may still be read by the grid queued before this one
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int rl = q * 32 + lane;  // accumulator row (TMEM lane)
        uint32_t tc_count = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++tc_count) {
            const int tile = u / ksplit;
            const int tw = tile % args.n_tiles_w;
            const int tn = tile / args.n_tiles_w;
            float* part = (ksplit > 1) ? args.partial + static_cast<int64_t>(u % ksplit) * args.M * args.ldo : nullptr;
            const int acc = tc_count & 1;
            const uint32_t aph = (tc_count >> 1) & 1u;
            // does any token of this tile carry a power of two?  The exponents are loaded before
            // the wait for the accumulator and first used after it, so their latency hides
            // behind the wait; almost always none is set.
            int tev[8];
            const bool has_exp = (MODE == kModeU) && args.row_exp != nullptr;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int64_t tk = static_cast<int64_t>(tn) * tile_n + 32 * c + lane;
                tev[c] = (has_exp && 32 * c + lane < tile_n && tk < args.M) ? args.row_exp[tk] : 0;
            }
            if (!(ok = tc::mbar_wait(acc_full(acc), aph, err))) break;
            const bool tile_scaled =
                has_exp && __any_sync(__activemask(), ((tev[0] | tev[1] | tev[2] | tev[3]) | (tev[4] | tev[5] | tev[6] | tev[7])) != 0);
            tc::tc_fence_after();
            const int64_t wrow = static_cast<int64_t>(tw) * kTileW + rl;
            const bool row_ok = wrow < args.rows_w;
            float scale = 1.0f;
            if (MODE == kModeU && row_ok) scale = f16_bits_to_float(args.s1[wrow]);
            const bool grad = (MODE == kModeU) && args.gpart != nullptr;
            double g = 0.0;
            for (int c0 = 0; c0 < tile_n; c0 += 32) {
                uint32_t v[32];
                tc::tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * 256 + c0, v);
                // the exponents of these 32 tokens: lane l loads token c0 + l's; almost always
                // all zero (rows inside fp16's range keep e = 0), and then the plain loop runs
                int el = 0;
                if (tile_scaled) {
                    const int64_t tk = static_cast<int64_t>(tn) * tile_n + c0 + lane;
                    el = (c0 + lane < tile_n && tk < args.M) ? args.row_exp[tk] : 0;
                }
                const bool scaled = tile_scaled && __any_sync(__activemask(), el != 0);
                tc::tmem_wait_ld();
                if (!scaled) {
                    if (row_ok) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int64_t tok = static_cast<int64_t>(tn) * tile_n + c0 + j;
                            if (c0 + j < tile_n && tok < args.M) {
                                const float f = __uint_as_float(v[j]);
                                if (grad) {
                                    g += static_cast<double>(bf16_bits_to_float(args.cot[tok * args.ldcot + wrow])) * f;
                                } else if (MODE == kModeU) {
                                    static_cast<uint16_t*>(args.out)[tok * args.ldo + wrow] = float_to_bf16_bits(scale * f);
                                } else if (part) {
                                    part[tok * args.ldo + wrow] = f;
                                } else {
                                    static_cast<uint16_t*>(args.out)[tok * args.ldo + wrow] =
                                        __half_as_ushort(__float2half_rn(f));
                                }
                            }
                        }
                    }
                } else if (MODE == kModeU) {
                    g += scaled_chunk(args, tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * 256 + c0, tn,
                                      tile_n, c0, wrow, row_ok, scale, grad, el);
                }
            }
            if (grad && row_ok) args.gpart[static_cast<int64_t>(tn) * args.rows_w + wrow] = g;
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

// Z[m][j] = fp16(bf16 x[m][j] * fp16 s2[j]) for j < d_in; row stride ldz.  Rows m by grid y;
// when d_in is a multiple of 8 (rows 16-byte aligned), up to VPT 16-byte vectors per thread,
// otherwise one element per thread.
__device__ __forceinline__ uint32_t scale2_f16(uint32_t xb2, uint32_t sh2) {
    const float a = bf16_bits_to_float(static_cast<uint16_t>(xb2 & 0xFFFFu)) * f16_bits_to_float(static_cast<uint16_t>(sh2 & 0xFFFFu));
    const float b = bf16_bits_to_float(static_cast<uint16_t>(xb2 >> 16)) * f16_bits_to_float(static_cast<uint16_t>(sh2 >> 16));
    return static_cast<uint32_t>(__half_as_ushort(__float2half_rn(a))) |
           (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(b))) << 16);
}

template <int VPT>
__global__ void __launch_bounds__(256) scale_convert_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ s2,
                                                           uint16_t* __restrict__ z, int64_t M, int64_t d_in, int64_t ldz) {
    pdl_wait();
    if ((d_in & 7) == 0) {
        // rows by grid y; each thread up to VPT 16-byte vectors of a row, loads issued together
        const int64_t per_row = d_in / 8;
        const int64_t step = static_cast<int64_t>(blockDim.x) * VPT;
        for (int64_t m = blockIdx.y; m < M; m += gridDim.y) {
            const uint4* xr = reinterpret_cast<const uint4*>(x + m * d_in);
            uint4* zr = reinterpret_cast<uint4*>(z + m * ldz);
            for (int64_t c0 = static_cast<int64_t>(blockIdx.x) * step + threadIdx.x; c0 < per_row;
                 c0 += static_cast<int64_t>(gridDim.x) * step) {
                uint4 xv[VPT], sv[VPT];
#pragma unroll
                for (int u = 0; u < VPT; ++u) {
                    const int64_t c = c0 + static_cast<int64_t>(u) * blockDim.x;
                    if (c < per_row) {
                        xv[u] = __ldcs(xr + c);
                        sv[u] = __ldg(reinterpret_cast<const uint4*>(s2) + c);
                    }
                }
#pragma unroll
                for (int u = 0; u < VPT; ++u) {
                    const int64_t c = c0 + static_cast<int64_t>(u) * blockDim.x;
                    if (c < per_row) {
                        uint4 o;
                        o.x = scale2_f16(xv[u].x, sv[u].x);
                        o.y = scale2_f16(xv[u].y, sv[u].y);
                        o.z = scale2_f16(xv[u].z, sv[u].z);
                        o.w = scale2_f16(xv[u].w, sv[u].w);
                        zr[c] = o;
                    }
                }
            }
        }
        return;
    }
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t m = blockIdx.y; m < M; m += gridDim.y) {
        const uint16_t* xr = x + m * d_in;
        uint16_t* zr = z + m * ldz;
        for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < d_in; j += stride) {
            const float v = bf16_bits_to_float(xr[j]) * f16_bits_to_float(s2[j]);
            zr[j] = __half_as_ushort(__float2half_rn(v));
        }
    }
}

// 2^k as a float for -126 <= k <= 127
__device__ __forceinline__ float pow2f(int k) { return __int_as_float((k + 127) << 23); }

// Row m of Z = fp16(2^-e_m x[m] (.) s2), with one power of two e_m per row: e_m = 0 while the row
// fits fp16 (L = sum_j |x_j s2_j| <= 2^14, and L / d_in >= 2^-10 so that typical values sit well
// inside fp16's normal range), else chosen so that 2^-e_m L <= 2^14.  Then every |Z| and every
// |T[m][k]| = |sum_j Z[m][j] V[j][k]| stays below fp16's largest value (65504) for any finite
// bf16 x and fp16 s2, and rows of small values keep their significant bits instead of falling
// into fp16's subnormals.  e_m goes to row_exp[m]; the epilogue of GEMM 2 multiplies by 2^e_m.
// Scaling by powers of two commutes with the roundings (bf16 x times fp16 s2 is exact in fp32;
// fp16 and fp32 round the same relative way wherever both values are normal).
// One block per row.  Pass 1 takes the largest |x| and L in fp32 (fixed order: per thread,
// then a tree).  Where that sum overflowed or fell below 2^-100 (rows of extreme magnitude), a
// second pass takes it again after scaling x by 2^-ex (2^ex <= max |x| < 2^(ex + 1)); values
// more than 2^126 below the row's largest flush to zero there, far below fp16's resolution of
// the row anyway.  The last pass converts.  Rows of up to 2048 kRowVecs values stay in
// registers; longer ones are read again from L2 for each pass.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float f16_lo(uint32_t h) { return f16_bits_to_float(static_cast<uint16_t>(h & 0xFFFFu)); }
__device__ __forceinline__ float f16_hi(uint32_t h) { return f16_bits_to_float(static_cast<uint16_t>(h >> 16)); }

template <int kRowVecs>
__global__ void __launch_bounds__(256) scale_convert_rows_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ s2,
                                                                uint16_t* __restrict__ z, int* __restrict__ row_exp,
                                                                int64_t M, int64_t d_in, int64_t ldz) {
    constexpr int kRowChunk = 256 * kRowVecs;  // vectors (of 8 values) per chunk
    pdl_wait();
    __shared__ unsigned int s_max[8];
    __shared__ float s_sum[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool vec = (d_in & 7) == 0;  // rows of whole 16-byte vectors (else one value at a time)
    const int64_t nvec = vec ? d_in / 8 : 0;
    const int64_t nchunk = vec ? (nvec + kRowChunk - 1) / kRowChunk : 0;
    const int lg = 64 - __clzll(static_cast<unsigned long long>(d_in - 1));  // ceil(log2 d_in)
    for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
        const uint16_t* xr = x + m * d_in;
        uint16_t* zr = z + m * ldz;
        uint4 xv[kRowVecs], sv[kRowVecs];
        auto load = [&](int64_t c) {
#pragma unroll
            for (int u = 0; u < kRowVecs; ++u) {
                const int64_t v = c * kRowChunk + u * 256 + tid;
                if (v < nvec) {
                    xv[u] = __ldg(reinterpret_cast<const uint4*>(xr) + v);
                    sv[u] = __ldg(reinterpret_cast<const uint4*>(s2) + v);
                } else {
                    xv[u] = make_uint4(0u, 0u, 0u, 0u);
                    sv[u] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
        };
        // ---- pass 1: the largest |x| (as bf16 bits, ordered like the magnitudes) and L
        unsigned int mx = 0u;
        float l1 = 0.0f;
        if (vec) {
            for (int64_t c = 0; c < nchunk; ++c) {
                load(c);
#pragma unroll
                for (int u = 0; u < kRowVecs; ++u) {
                    const uint32_t w[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
                    const uint32_t h[4] = {sv[u].x, sv[u].y, sv[u].z, sv[u].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        mx = max(mx, max(w[q] & 0x7FFFu, (w[q] >> 16) & 0x7FFFu));
                        l1 += fabsf(bf16_lo(w[q]) * f16_lo(h[q])) + fabsf(bf16_hi(w[q]) * f16_hi(h[q]));
                    }
                }
            }
        } else {
            for (int64_t j = tid; j < d_in; j += 256) {
                mx = max(mx, static_cast<unsigned int>(xr[j] & 0x7FFFu));
                l1 += fabsf(bf16_bits_to_float(xr[j]) * f16_bits_to_float(s2[j]));
            }
        }
        mx = __reduce_max_sync(0xffffffffu, mx);
        for (int off = 16; off > 0; off >>= 1) l1 += __shfl_xor_sync(0xffffffffu, l1, off);
        if (lane == 0) {
            s_max[warp] = mx;
            s_sum[warp] = l1;
        }
        __syncthreads();
        mx = 0u;
        l1 = 0.0f;
        for (int w = 0; w < 8; ++w) {
            mx = max(mx, s_max[w]);
            l1 += s_sum[w];
        }
        __syncthreads();  // s_max and s_sum are written again below or by the next row
        const bool finite_row = mx != 0u && mx < 0x7F80u;  // neither all zero nor inf/NaN
        // the conversion multiplies x by f1 f2, then by s2, then by fs (exact powers of two)
        float f1 = 1.0f, f2 = 1.0f, fs = 1.0f;
        int e = 0;
        if (finite_row && l1 > 0.0f) {
            if (l1 <= 3.0e38f && l1 >= 0x1p-100f) {
                int c = 0;
                frexpf(l1, &c);  // L < 2^c
                const bool fits = (c <= 14) && (c - 1 - lg >= -10);
                if (!fits) {
                    e = c - 14;  // |e| <= 114
                    fs = pow2f(-e);
                }
            } else {
                // ---- pass 2 (rows of extreme magnitude): L after scaling x by 2^-ex
                const int ex = (mx >= 0x80u) ? static_cast<int>(mx >> 7) - 127 : (31 - __clz(mx)) - 133;
                f1 = pow2f((-ex) / 2);
                f2 = pow2f(-ex - (-ex) / 2);  // 2^-ex = f1 f2, each a normal float
                float l2 = 0.0f;
                if (vec) {
                    for (int64_t c = 0; c < nchunk; ++c) {
                        if (nchunk > 1) load(c);
#pragma unroll
                        for (int u = 0; u < kRowVecs; ++u) {
                            const uint32_t w[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
                            const uint32_t h[4] = {sv[u].x, sv[u].y, sv[u].z, sv[u].w};
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                l2 += fabsf(bf16_lo(w[q]) * f1 * f2 * f16_lo(h[q])) + fabsf(bf16_hi(w[q]) * f1 * f2 * f16_hi(h[q]));
                        }
                    }
                } else {
                    for (int64_t j = tid; j < d_in; j += 256)
                        l2 += fabsf(bf16_bits_to_float(xr[j]) * f1 * f2 * f16_bits_to_float(s2[j]));
                }
                for (int off = 16; off > 0; off >>= 1) l2 += __shfl_xor_sync(0xffffffffu, l2, off);
                if (lane == 0) s_sum[warp] = l2;
                __syncthreads();
                l2 = 0.0f;
                for (int w = 0; w < 8; ++w) l2 += s_sum[w];
                __syncthreads();
                if (l2 > 0.0f) {
                    int c = 0;
                    frexpf(l2, &c);  // l2 < 2^c <= 2^38 (d_in values of |2^-ex x| < 2, |s2| <= 65504)
                    const int sh = min(14 - c, 127);  // a smaller sh keeps the bound (sums below 2^-113 only)
                    e = ex - sh;
                    fs = pow2f(sh);
                } else {
                    f1 = f2 = 1.0f;  // nothing survived the scaling: the row converts as it is
                }
            }
        }
        if (tid == 0) row_exp[m] = e;
        // ---- conversion: z = fp16(((x f1 f2) s2) fs)
        if (vec) {
            for (int64_t c = 0; c < nchunk; ++c) {
                if (nchunk > 1) load(c);
#pragma unroll
                for (int u = 0; u < kRowVecs; ++u) {
                    const int64_t v = c * kRowChunk + u * 256 + tid;
                    if (v < nvec) {
                        const uint32_t w[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
                        const uint32_t h[4] = {sv[u].x, sv[u].y, sv[u].z, sv[u].w};
                        uint32_t o[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float a = (bf16_lo(w[q]) * f1 * f2) * f16_lo(h[q]) * fs;
                            const float b = (bf16_hi(w[q]) * f1 * f2) * f16_hi(h[q]) * fs;
                            o[q] = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(a))) |
                                   (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(b))) << 16);
                        }
                        reinterpret_cast<uint4*>(zr)[v] = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
        } else {
            for (int64_t j = tid; j < d_in; j += 256) {
                const float v = (bf16_bits_to_float(xr[j]) * f1 * f2) * f16_bits_to_float(s2[j]) * fs;
                zr[j] = __half_as_ushort(__float2half_rn(v));
            }
        }
    }
}

// T[m][k] = fp16( sum over splits s = 0 .. S-1, in order, of partial[s][m][k] ) for k < r;
// four k per thread (r % 32 == 0 and ldt % 8 == 0: 16-byte loads, 8-byte stores).
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ partial, int S, int64_t M,
                                                           int64_t r, int64_t ldt, uint16_t* __restrict__ t) {
    pdl_wait();
    const int64_t per_row = r / 4;
    const int64_t n = M * per_row;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = e / per_row, k = (e - m * per_row) * 4;
        float4 acc = *reinterpret_cast<const float4*>(partial + m * ldt + k);
        for (int sp = 1; sp < S; ++sp) {
            const float4 v = *reinterpret_cast<const float4*>(partial + (static_cast<int64_t>(sp) * M + m) * ldt + k);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        uint2 o;
        o.x = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(acc.x))) |
              (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(acc.y))) << 16);
        o.y = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(acc.z))) |
              (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(acc.w))) << 16);
        *reinterpret_cast<uint2*>(t + m * ldt + k) = o;
    }
}

// grad[i] = sum over token tiles tn (in order) of gpart[tn][i], fp64, rounded to fp32.
__global__ void __launch_bounds__(256) grad_reduce_kernel(const double* __restrict__ gpart, int64_t n_tiles,
                                                         int64_t rows, float* __restrict__ grad) {
    pdl_wait();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < rows;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        double g = 0.0;
        for (int64_t tn = 0; tn < n_tiles; ++tn) g += gpart[tn * rows + i];
        grad[i] = static_cast<float>(g);
    }
}

}  // namespace nq

// ------------------------------------------------------------------------------ host side
#include <atomic>

namespace {

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

struct PrefillPlan {
    int64_t ldz, ldt;
    int tile_n1, tile_n2;  // token tiles of GEMM 1 and GEMM 2
    int ksplit1;           // K splits of GEMM 1 (when its packed signs arrive by TMA)
    size_t off_z, off_t, off_p, off_g, off_e, total;
};

// K splits for a GEMM of `tiles` output tiles over nkb k blocks: the fewest k-block steps on
// the busiest SM, counted as waves x (k blocks per unit + 2 for the unit's pipeline fill and
// drain), plus the fp32 partials' extra traffic (written once, read once; about 2.25 MB per
// k-block step of time).  Every unit keeps at least 4 k blocks.
int choose_ksplit(int64_t tiles, int64_t nkb, int64_t M, int64_t r, int sms) {
    int best = 1;
    double best_cost = -1.0;
    const int64_t top = std::min<int64_t>(16, nkb / 4);
    for (int64_t S = 1; S <= std::max<int64_t>(1, top); ++S) {
        const int64_t waves = (tiles * S + sms - 1) / sms;
        const int64_t per = (nkb + S - 1) / S;
        const double extra = (S > 1) ? static_cast<double>(S) * M * r * 8 / 2.25e6 : 0.0;
        const double cost = static_cast<double>(waves * (per + 2)) + extra;
        if (best_cost < 0.0 || cost < best_cost) {
            best_cost = cost;
            best = static_cast<int>(S);
        }
    }
    return best;
}

// Tokens per tile (MMA N, a multiple of 16 up to 256) for a GEMM with n_tiles_w weight tiles:
// the fewest waves of persistent tiles over the SMs, each wave costing about max(N, 192) + 64
// (the weight expansion puts a floor under a stage's time; splitting N below it buys nothing).
// Ties go to the larger N.
int choose_tile_n(int64_t n_tiles_w, int64_t M, int sms) {
    int best = 16;
    int64_t best_cost = -1;
    const int top = static_cast<int>(std::min<int64_t>(256, round_up(M, 16)));
    for (int tn = 16; tn <= top; tn += 16) {
        const int64_t tiles = n_tiles_w * ((M + tn - 1) / tn);
        const int64_t waves = (tiles + sms - 1) / sms;
        const int64_t cost = waves * (std::max(tn, 192) + 64);
        if (best_cost < 0 || cost <= best_cost) {
            best_cost = cost;
            best = tn;
        }
    }
    return best;
}

PrefillPlan plan_prefill(const nq_lrb_layer* L, int64_t M) {
    PrefillPlan p{};
    const int sms = nq_host::sm_count();
    p.tile_n1 = choose_tile_n((L->r + nq::kTileW - 1) / nq::kTileW, M, sms);
    p.tile_n2 = choose_tile_n((L->d_out + nq::kTileW - 1) / nq::kTileW, M, sms);
    p.ldz = round_up(L->d_in, 8);  // 16-byte aligned rows for TMA
    p.ldt = round_up(L->r, 8);
    p.off_z = NQ_WS_HEADER_BYTES;  // past the reserved workspace header
    p.off_t = p.off_z + align256(static_cast<size_t>(M * p.ldz) * 2);
    p.off_p = p.off_t + align256(static_cast<size_t>(M * p.ldt) * 2);
    const int64_t tiles1 = ((L->r + nq::kTileW - 1) / nq::kTileW) * ((M + p.tile_n1 - 1) / p.tile_n1);
    p.ksplit1 = choose_ksplit(tiles1, (L->d_in + nq::kTileK - 1) / nq::kTileK, M, L->r, sms);
    p.off_g = p.off_p + (p.ksplit1 > 1 ? align256(static_cast<size_t>(p.ksplit1) * M * p.ldt * 4) : 0);
    // gradient mode: fp64 partial per (token tile of GEMM 2, row)
    const int64_t n_tn2 = (M + p.tile_n2 - 1) / p.tile_n2;
    p.off_e = p.off_g + align256(static_cast<size_t>(n_tn2 * L->d_out) * sizeof(double));
    p.total = p.off_e + align256(static_cast<size_t>(M) * sizeof(int));  // per-token exponents
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

// 2-D uint32 tensor [rows][ld] of packed signs (nwords valid words per row); box = kBitsWords
// words x box_rows.  Needs a 16-byte aligned base and row stride; false when not encodable.
bool make_tmap_bits(CUtensorMap* map, const uint32_t* base, int64_t rows, int64_t nwords, int64_t ld, int box_rows) {
    auto enc = get_encode();
    if (!enc || (ld % 4) != 0 || (reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(nwords), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 4)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(nq::kBitsWords), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kUmmaSmemBudget = 220 * 1024;

size_t umma_stage_bytes(int tile_n) {
    const size_t b = static_cast<size_t>(tile_n) * nq::kTileK * 2;
    return nq::kABytes + ((b + 1023) & ~static_cast<size_t>(1023)) + nq::kBitsBytes;
}

size_t umma_smem_bytes(int tile_n, int stages) {
    return 1024 /* alignment slack */ + stages * umma_stage_bytes(tile_n) + 8 * (3 * nq::kMaxStages + 6) + 16;
}

// As many stages as fit the budget: narrow tiles run short stages, and the ring must cover the
// latency of a tile's TMA load (about a microsecond) to keep the tensor core fed.
int umma_stages(int tile_n) {
    int st = nq::kMaxStages;
    while (st > 2 && umma_smem_bytes(tile_n, st) > kUmmaSmemBudget) --st;
    return st;
}

template <int MODE, bool SPLIT>
nq_status launch_umma_t(const nq::PrefillArgs& a, const CUtensorMap& map, const CUtensorMap& bits_map,
                        cudaStream_t stream, bool pdl) {
    static std::atomic<bool> attr_done[64];  // per device; setting an attribute twice is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    const size_t smem = kUmmaSmemBudget;
    if (dev >= 0 && dev < 64 && !attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(nq::lrb_umma_kernel<MODE, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return NQ_ERR_LAUNCH;
        attr_done[dev].store(true, std::memory_order_release);
    }
    const int units = a.n_tiles_w * a.n_tiles_n * ((MODE == nq::kModeV && a.ksplit > 1) ? a.ksplit : 1);
    int grid = nq_host::sm_count();
    if (grid > units) grid = units;
    nq::PrefillArgs args = a;
    args.stages = umma_stages(a.tile_n);
    CUtensorMap tm = map, tb = bits_map;
    void* kargs[] = {&tm, &tb, &args};
    return nq_host::launch_pdl(reinterpret_cast<const void*>(nq::lrb_umma_kernel<MODE, SPLIT>), dim3(grid),
                               dim3(nq::kPrefillThreads), umma_smem_bytes(a.tile_n, args.stages), stream, kargs,
                               pdl) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_LAUNCH;
}

template <int MODE>
nq_status launch_umma(const nq::PrefillArgs& a, const CUtensorMap& map, const CUtensorMap& bits_map, cudaStream_t stream,
                      bool pdl) {
    if constexpr (MODE == nq::kModeV) {
        if (a.ksplit > 1) return launch_umma_t<MODE, true>(a, map, bits_map, stream, pdl);
    }
    return launch_umma_t<MODE, false>(a, map, bits_map, stream, pdl);
}

}  // namespace

namespace nq_host {
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() { return get_encode(); }
}  // namespace nq_host

size_t nq_prefill_workspace_bytes(const nq_lrb_layer* L, int64_t M) { return plan_prefill(L, M).total; }

namespace {

// Z = fp16(x . s2) and T = fp16(Z V) of layer L into the workspace ws, laid out by plan p.
nq_status launch_stage1(const nq_lrb_layer* L, const uint16_t* x, int64_t M, void* ws, const PrefillPlan& p,
                        cudaStream_t stream, bool pdl, int* row_exp = nullptr) {
    uint16_t* z = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + p.off_z);
    uint16_t* t = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + p.off_t);
    unsigned int* err = nq_host::error_word();
    if (row_exp) {  // Z = fp16(2^-e_m x * s2), one exponent per token
        const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(M, 65535));
        const uint16_t* s2 = L->s2;
        int64_t d_in = L->d_in, ldz = p.ldz;
        void* args[] = {&x, &s2, &z, &row_exp, &M, &d_in, &ldz};
        // four vectors per thread: rows of up to 8192 values stay in registers, longer ones are
        // read again (from L2) by the later passes; a small footprint keeps several blocks per SM
        const void* fn = reinterpret_cast<const void*>(nq::scale_convert_rows_kernel<4>);
        if (nq_host::launch_pdl(fn, dim3(blocks), dim3(256), 0, stream, args, pdl) != cudaSuccess)
            return NQ_ERR_LAUNCH;
    } else {  // Z = fp16(x * s2)
        // four vectors per thread once the job has enough of them for 2 blocks per SM at that
        // depth; one otherwise (more, smaller blocks for few rows)
        const int64_t per_row = (L->d_in % 8 == 0) ? L->d_in / 8 : L->d_in;  // work items per row
        const bool deep = (L->d_in % 8 == 0) && M * per_row >= 2LL * 1024 * nq_host::sm_count();
        const int64_t per_block = deep ? 1024 : 256;
        const unsigned gx = static_cast<unsigned>(std::min<int64_t>((per_row + per_block - 1) / per_block, 64));
        const unsigned gy = static_cast<unsigned>(std::min<int64_t>(M, 65535));
        const uint16_t* s2 = L->s2;
        int64_t d_in = L->d_in, ldz = p.ldz;
        void* args[] = {&x, &s2, &z, &M, &d_in, &ldz};
        const void* fn = deep ? reinterpret_cast<const void*>(nq::scale_convert_kernel<4>)
                              : reinterpret_cast<const void*>(nq::scale_convert_kernel<1>);
        if (nq_host::launch_pdl(fn, dim3(gx, gy), dim3(256), 0, stream,
                                args, pdl) != cudaSuccess)
            return NQ_ERR_LAUNCH;
    }
    {  // T = fp16(Z V): weights = V^T (M-extent r, K = d_in), B = Z
        const int tile_n = p.tile_n1;
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
        CUtensorMap bmap;
        std::memset(&bmap, 0, sizeof(bmap));
        a.bits_tma = make_tmap_bits(&bmap, L->V, L->d_in, L->r / 32, L->ldv, nq::kTileK) ? 1 : 0;
        a.ksplit = a.bits_tma ? p.ksplit1 : 1;
        a.partial = a.ksplit > 1 ? reinterpret_cast<float*>(static_cast<char*>(ws) + p.off_p) : nullptr;
        nq_status st = launch_umma<nq::kModeV>(a, map, bmap, stream, pdl);
        if (st != NQ_OK || a.ksplit == 1) return st;
        // T = fp16 of the splits' sum, in split order
        const float* part = a.partial;
        int S = a.ksplit;
        int64_t r = L->r, ldt = p.ldt;
        const int64_t items = M * (r / 4);
        const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((items + 255) / 256, 8LL * nq_host::sm_count()));
        void* args[] = {&part, &S, &M, &r, &ldt, &t};
        return nq_host::launch_pdl(reinterpret_cast<const void*>(nq::splitk_reduce_kernel), dim3(blocks), dim3(256), 0,
                                   stream, args, pdl) == cudaSuccess
                   ? NQ_OK
                   : NQ_ERR_LAUNCH;
    }
}

}  // namespace

void nq_prefill_stage1_layout(const nq_lrb_layer* L, int64_t M, size_t* off_z, int64_t* ldz, size_t* off_t,
                              int64_t* ldt, size_t* bytes) {
    const PrefillPlan p = plan_prefill(L, M);
    *off_z = p.off_z;
    *ldz = p.ldz;
    *off_t = p.off_t;
    *ldt = p.ldt;
    *bytes = p.off_g;
}

nq_status nq_launch_prefill_stage1(const nq_lrb_layer* L, const uint16_t* x, int64_t M, void* ws, cudaStream_t stream,
                                   bool pdl) {
    return launch_stage1(L, x, M, ws, plan_prefill(L, M), stream, pdl);
}

nq_status nq_launch_prefill(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                            cudaStream_t stream, bool pdl, const uint16_t* cot, float* grad) {
    const PrefillPlan p = plan_prefill(L, M);
    uint16_t* t = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + p.off_t);
    unsigned int* err = nq_host::error_word();
    int* row_exp = reinterpret_cast<int*>(static_cast<char*>(ws) + p.off_e);
    nq_status st0 = launch_stage1(L, x, M, ws, p, stream, pdl, row_exp);
    if (st0 != NQ_OK) return st0;
    {  // Y = bf16(s1 * (T U^T)): weights = U (M-extent d_out, K = r), B = T
        const int tile_n = p.tile_n2;
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
        a.row_exp = row_exp;
        a.err = err;
        double* gpart = reinterpret_cast<double*>(static_cast<char*>(ws) + p.off_g);
        if (grad) {
            a.out = nullptr;
            a.cot = cot;
            a.ldcot = L->d_out;
            a.gpart = gpart;
        }
        CUtensorMap bmap;
        std::memset(&bmap, 0, sizeof(bmap));
        a.bits_tma = make_tmap_bits(&bmap, L->U, L->d_out, L->r / 32, L->ldu, nq::kTileW) ? 1 : 0;
        nq_status st = launch_umma<nq::kModeU>(a, map, bmap, stream, pdl);
        if (st != NQ_OK) return st;
        if (grad) {  // sum the token tiles' partials per row, in order
            int64_t n_tiles = a.n_tiles_n, rows = L->d_out;
            const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((rows + 255) / 256, 4LL * nq_host::sm_count()));
            void* args[] = {&gpart, &n_tiles, &rows, &grad};
            if (nq_host::launch_pdl(reinterpret_cast<const void*>(nq::grad_reduce_kernel), dim3(blocks), dim3(256), 0,
                                    stream, args, pdl) != cudaSuccess)
                return NQ_ERR_LAUNCH;
        }
    }
    return NQ_OK;
}
