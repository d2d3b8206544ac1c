// decode_stream.cu -- decode (batch 1..2) of one LRB layer, or of up to four layers that share
// their input, as ONE persistent launch with one CTA per SM.
//
// Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models"
// (research.samsung.com blog), section 2, factorisation equation, evaluated right to left from
// the packed signs; section 4, "Inference Performance", names this binary GEMV for decoding.
//
//   stage 1:  t[m][k] = sum_j V_jk z[m][j],   z = s2 (.) x        (reduction over d_in)
//   stage 2:  y[m][i] = bf16( s1_i sum_k U_ik t[m][k] )           (reduction over r)
//
// Roles.  Warp 0 is the producer: one lane streams this CTA's share of the packed words, first
// its stage-1 tiles of V, then its stage-2 row blocks of U, by TMA into a ring of shared-memory
// slots, and never waits for activations -- weights do not depend on the previous kernel, so the
// stream starts at the first instruction and keeps running while the consumers wait for x, sit
// at the grid barrier or build tables.  Warps 1..8 consume: stage 1, a bounded grid barrier
// (every CTA is resident: one CTA per SM, grid <= SM count), stage 2.
//
// Arithmetic.  Both stages multiply the packed bits, masked per bit offset, as the u8 A operand
// of mma.sync m16n8k32 with three signed base-256 digits of a 23-bit fixed-point activation as
// the s8 B operand, so every product sum is an exact integer.
//  - z is quantised per run (the rows one CTA reduces for one 16-word column chunk), with a
//    shift from the run's own maximum, clamped to a common exponent Q per batch row and layer
//    (Q = 16 + the shift of the bound max|s2| max|x|, which every CTA computes identically).  A
//    run's partial of t, (2 P - sum z_q) 2^(Q - shift), is then an exact integer at the common
//    scale 2^-Q and is added into t's int64 accumulator in the workspace with integer atomics:
//    exact and independent of order.
//  - Stage 2 reads the whole accumulator, takes its maximum and re-quantises t to 23 bits
//    (round to nearest even), so y = s1 (2 P - sum t_q) 2^(d - Q) up to the final bf16 rounding.
//
// Workspace.  The grid-barrier counter, the bounds on |t| and the accumulators live in the
// workspace's leading region, which must be zero before the first call.  The counter only grows
// (each launch of G CTAs adds G), so counter / G numbers the launches; the accumulators and
// bounds come in two halves, launch k uses half k & 1 and clears the other one, which launch
// k - 1 read and launch k + 1 will use.
#include "tc_common.cuh"

namespace nq {
namespace ds {

constexpr int kCW = 8;                   // consumer warps
constexpr int kThreads = 32 * (kCW + 1);
constexpr int kTileWords = 16;           // words per stage-1 tile row: 64-byte rows
constexpr int kMaxM = 2;                 // batch rows: three digit columns each in one 8-wide N tile
constexpr int kMaxMem = NQ_MAX_GROUP;
constexpr int kMaxSlots = 16;
constexpr int kMaxTiles1 = 64;           // stage-1 tiles per CTA (runs are at most as many)
constexpr int kTPer = 16;                // accumulator values a consumer thread loads at once (stage 2's prologue)
constexpr int kZoneHalf = NQ_WS_ZONE_BYTES / 16;  // int64 elements per zone half

struct Member {
    CUtensorMap tmV;  // V words [d_in][nw] (row stride ldv), box {16, H1}, 64-byte swizzle
    CUtensorMap tmU;  // U words [d_out][nw] (row stride ldu), box {BW, R2}
    const uint16_t* s1;
    const uint16_t* s2;
    uint16_t* y;       // [M][d_out]
    int tacc;          // [M][rp] exact accumulator of t (units of 2^-Q): element offset in a zone half
    int d_out, r, nw, ng;  // ng = 8-word groups of a U row
    int BW, R2;        // stage-2 box: BW words (= 8 or 24 mod 32) by R2 rows
    int rp;            // r rounded up to a chunk (512)
    int nchunks;       // 16-word chunks of a V row
    int btab;          // byte offset of t's digit table in shared memory
    long long b2_bytes;  // bytes of one stage-2 block
};

struct Params {
    Member mem[kMaxMem];
    const uint16_t* x;
    unsigned long long* sync;  // [0] grid-barrier arrivals, [1] arrivals after reading t
    unsigned int* err;
    int nmem, M, d_in, H1, nrb, ns, slot_bytes;
    int t1_off[kMaxMem + 1];   // first stage-1 tile of each member (tiles: member, chunk, row block)
    int t2_off[kMaxMem + 1];   // first stage-2 block of each member
    long long b2_cum[kMaxMem + 1];  // bytes of the stage-2 blocks before each member
    long long* zone;           // two halves of kZoneHalf int64: launch k accumulates into half k & 1
    int off_tq;                // t_q of the members, int32 [M][r], while the digit tables are built
    int n1max, n2max, R2max;   // per-CTA table sizes
    int off_ztab, off_zs, off_s2s, off_s1s, off_dw;  // dynamic shared memory carve-up
};

// ------------------------------------------------------------------ small device helpers
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kCW) : "memory"); }

__device__ __forceinline__ void mbar_arrive_cnt(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// balanced base-256 digits of a 23-bit signed integer, as s8 bytes
__device__ __forceinline__ void digits3(int v, uint32_t& d0, uint32_t& d1, uint32_t& d2) {
    const int a0 = (v << 24) >> 24;
    const int v1 = (v - a0) >> 8;
    const int a1 = (v1 << 24) >> 24;
    const int a2 = (v1 - a1) >> 8;
    d0 = static_cast<uint32_t>(a0) & 255u;
    d1 = static_cast<uint32_t>(a1) & 255u;
    d2 = static_cast<uint32_t>(a2) & 255u;
}

// 4x4 byte transpose of four rows given in the order (w0, w1, w2, w3): o[b] holds byte b of the
// four rows, row order chosen by the selectors of the last step: (0x5410, 0x7632) keeps the
// given order; (0x4105, 0x6327) undoes a rotation by one (w0..w3 = rows 1, 2, 3, 0).
__device__ __forceinline__ void transpose_rows(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, uint32_t sel_lo,
                                               uint32_t sel_hi, uint32_t (&o)[4]) {
    const uint32_t t0 = __byte_perm(w0, w1, 0x5140);  // w0.b0 w1.b0 w0.b1 w1.b1
    const uint32_t t1 = __byte_perm(w0, w1, 0x7362);  // w0.b2 w1.b2 w0.b3 w1.b3
    const uint32_t t2 = __byte_perm(w2, w3, 0x5140);
    const uint32_t t3 = __byte_perm(w2, w3, 0x7362);
    o[0] = __byte_perm(t0, t2, sel_lo);
    o[1] = __byte_perm(t0, t2, sel_hi);
    o[2] = __byte_perm(t1, t3, sel_lo);
    o[3] = __byte_perm(t1, t3, sel_hi);
}

// Stage-1 slot layout.  TMA writes the tile [H1 rows][16 words] with the 64-byte swizzle: the
// 16-byte unit p of row j lands at unit p ^ ((j >> 1) & 3).  The consumers then transpose in
// place: the thread of quad q (rows 4q..4q+3) and unit p reads those 16 words (row 4q + i in a
// rotated order, i + (q & 1)) and writes back T[q][w] for its four words w = 4p + a, where
// T[q][w][b] holds byte b of word w of the quad's four rows, into row 4q + (a ^ (q & 3)), unit
// p of its own region.  Both passes and the MMA reads below are free of shared-memory bank
// conflicts.
__device__ __forceinline__ uint32_t s1_unit_addr(uint32_t slot, int row, int unit) {
    return slot + static_cast<uint32_t>(row * 64 + ((unit ^ ((row >> 1) & 3)) << 4));
}
// address of T[q][w]
__device__ __forceinline__ uint32_t s1_T_addr(uint32_t slot, int q, int w) {
    return s1_unit_addr(slot, 4 * q + ((w & 3) ^ (q & 3)), w >> 2);
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

// member of a global index from prefix offsets
__device__ __forceinline__ int member_of(const int* off, int n, int idx) {
    int l = 0;
    while (l + 1 < n && idx >= off[l + 1]) ++l;
    return l;
}

// First stage-2 block of CTA b: blocks are split in proportion to their bytes.
__device__ __forceinline__ int stage2_start(const Params& P, int b, int G) {
    const long long total = P.b2_cum[P.nmem];
    const long long target = (total * b + G - 1) / G;  // first byte owned by CTA b
    for (int l = 0; l < P.nmem; ++l) {
        if (target < P.b2_cum[l + 1]) {
            const long long rel = target - P.b2_cum[l];
            const long long blk = (rel + P.mem[l].b2_bytes - 1) / P.mem[l].b2_bytes;
            return P.t2_off[l] + static_cast<int>(blk);
        }
    }
    return P.t2_off[P.nmem];
}

// Sums the digit columns of one output row into P_m = D(3m) + 2^8 D(3m+1) + 2^16 D(3m+2) for
// m = 0, 1.  Lane tig holds columns 2 tig (c_lo) and 2 tig + 1 (c_hi); the result is returned
// in every lane of the quad.
__device__ __forceinline__ void combine_cols(int c_lo, int c_hi, int tig, long long& P0, long long& P1) {
    long long p0 = 0, p1 = 0;
    if (tig == 0) p0 = static_cast<long long>(c_lo) + (static_cast<long long>(c_hi) << 8);
    if (tig == 1) {
        p0 = static_cast<long long>(c_lo) << 16;
        p1 = static_cast<long long>(c_hi);
    }
    if (tig == 2) p1 = (static_cast<long long>(c_lo) << 8) + (static_cast<long long>(c_hi) << 16);
    p0 += __shfl_xor_sync(0xffffffffu, p0, 1);
    p1 += __shfl_xor_sync(0xffffffffu, p1, 1);
    p0 += __shfl_xor_sync(0xffffffffu, p0, 2);
    p1 += __shfl_xor_sync(0xffffffffu, p1, 2);
    P0 = p0;
    P1 = p1;
}

__device__ __forceinline__ double pow2_d(int e) { return __longlong_as_double(static_cast<long long>(1023 + e) << 52); }

// Exponent e of a positive float v = f 2^e with 0.5 <= f < 1, from its bits (frexp for
// subnormals, which stage 1 meets only for values below 2^-126).
__device__ __forceinline__ int exp_of(float v) {
    const int biased = static_cast<int>((__float_as_uint(v) >> 23) & 0xffu);
    if (biased != 0) return biased - 126;
    int e = 0;
    frexpf(v, &e);
    return e;
}

// End of a stage-1 run (member mb, chunk c): this warp's exact partials of t for its 64
// outputs, (2 P - sum z_q) 2^(Q - shift), into the accumulator; the warp's sums restart at 0.
// The digit columns are combined into P in registers and parked in the warp's buffer pbuf
// ([64 outputs][2 batch rows]); a short rolled loop then adds them to the accumulator, two
// outputs per lane.
__device__ __forceinline__ void flush_run(const Member& mb, long long* half, int c, int cw, int lane, int M,
                                          long long zsum0, long long zsum1, const int* sh, const int* Q,
                                          int (&acc)[2][2][4], long long* pbuf) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int wi = 0; wi < 2; ++wi)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int rh = 0; rh < 2; ++rh) {
                long long P0, P1;
                combine_cols(acc[wi][h][2 * rh] >> gid, acc[wi][h][2 * rh + 1] >> gid, tig, P0, P1);
                const int kl = 32 * wi + 16 * h + 8 * rh + gid;
                if (tig == 0) pbuf[2 * kl] = P0;
                if (tig == 1) pbuf[2 * kl + 1] = P1;
            }
    __syncwarp();
#pragma unroll 1
    for (int e = lane; e < 64 * M; e += 32) {
        const int m = e >> 6, kl = e & 63;
        const int k = 512 * c + 64 * cw + kl;
        if (k < mb.r) {
            const long long v = (2 * pbuf[2 * kl + m] - (m ? zsum1 : zsum0)) << (Q[m] - sh[m]);
            atomicAdd(reinterpret_cast<unsigned long long*>(half + mb.tacc + static_cast<int64_t>(m) * mb.rp + k),
                      static_cast<unsigned long long>(v));
        }
    }
    __syncwarp();
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[a][b][e] = 0;
}

// Sum over the lanes of aligned groups of `width` lanes (a power of two <= 32).
__device__ __forceinline__ long long group_sum(long long v, int width) {
    for (int off = 1; off < width; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// ------------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(kThreads, 1) decode_stream_kernel(const __grid_constant__ Params P) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kMaxSlots];
    __shared__ __align__(8) uint64_t empty_bar[kMaxSlots];
    __shared__ unsigned int s_s2max[kMaxMem];              // max |s2| per member (float bits)
    __shared__ unsigned int s_xmax[kMaxM];                 // max |x| per batch row (float bits)
    __shared__ int s_Q[kMaxMem][kMaxM];                    // common exponent of t's accumulator
    __shared__ unsigned int s_tilemax[kMaxTiles1][kMaxM];  // max |z| per stage-1 tile (float bits)
    __shared__ int s_tilesh[kMaxTiles1][kMaxM];            // shift of the tile's run
    __shared__ long long s_tilezsum[kMaxTiles1][kMaxM];    // sum of z_q over the tile's rows
    __shared__ long long s_tilezabs[kMaxTiles1][kMaxM];    // sum of |z_q|
    __shared__ int s_td[kMaxMem][kMaxM];                   // right shift of t's accumulator
    __shared__ long long s_tsum[kMaxMem][kMaxM];           // sum over k of t_q
    __shared__ unsigned char s_tl[kMaxTiles1];             // member of each stage-1 tile
    __shared__ short s_tc[kMaxTiles1], s_trb[kMaxTiles1];  // chunk and row block
    __shared__ unsigned char s_rfirst[kMaxTiles1], s_rlast[kMaxTiles1];  // first / last tile of its run
    __shared__ volatile int s_abort;
    __shared__ int s_issued;
    __shared__ unsigned long long s_launch;  // index of this launch on the workspace

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int G = gridDim.x, cta = blockIdx.x;
    const int M = P.M, ns = P.ns;
    const int T1 = P.t1_off[P.nmem];
    const int a1 = static_cast<int>(static_cast<long long>(T1) * cta / G);
    const int n1 = static_cast<int>(static_cast<long long>(T1) * (cta + 1) / G) - a1;
    const int a2 = stage2_start(P, cta, G);
    const int n2 = stage2_start(P, cta + 1, G) - a2;
    const int KS = P.H1 / 32;  // K steps (32 rows) per stage-1 tile
    // per zone half: [member][m] sums |z_q| 2^(Q - shift), exact bounds on |t| at scale 2^-Q
    long long* const bounds_base = reinterpret_cast<long long*>(P.sync + 8);

    // 1024-byte aligned base (the swizzled TMA boxes need it)
    const uint32_t raw_base = tc::smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    unsigned char* const gbase = smem_raw + (base - raw_base);
    auto full = [&](int s) { return tc::smem_u32(&full_bar[s]); };
    auto empty = [&](int s) { return tc::smem_u32(&empty_bar[s]); };
    auto slot_addr = [&](int s) { return base + static_cast<uint32_t>(s * P.slot_bytes); };

    if (tid == 0) {
        for (int s = 0; s < ns; ++s) {
            tc::mbar_init(full(s), 1);
            tc::mbar_init(empty(s), kCW);
        }
        tc::mbar_fence_init();
        s_abort = 0;
        s_issued = 0;
    }
    // stage-1 tiles of this CTA: member, chunk, row block, and the run (consecutive tiles of
    // one member and chunk) each belongs to
    if (tid < n1) {
        const int t = tid;
        auto key = [&](int u, int& l, int& c, int& rb) {
            const int g = a1 + u;
            l = member_of(P.t1_off, P.nmem, g);
            const int loc = g - P.t1_off[l];
            c = loc / P.nrb;
            rb = loc - c * P.nrb;
        };
        int l, c, rb;
        key(t, l, c, rb);
        s_tl[t] = static_cast<unsigned char>(l);
        s_tc[t] = static_cast<short>(c);
        s_trb[t] = static_cast<short>(rb);
        int f = t, e = t;
        while (f > 0) {
            int l2, c2, rb2;
            key(f - 1, l2, c2, rb2);
            if (l2 != l || c2 != c) break;
            --f;
        }
        while (e + 1 < n1) {
            int l2, c2, rb2;
            key(e + 1, l2, c2, rb2);
            if (l2 != l || c2 != c) break;
            ++e;
        }
        s_rfirst[t] = static_cast<unsigned char>(f);
        s_rlast[t] = static_cast<unsigned char>(e);
    }
    if (tid < kMaxMem) s_s2max[tid] = 0u;
    if (tid < kMaxM) s_xmax[tid] = 0u;
    for (int e = tid; e < kMaxTiles1 * kMaxM; e += kThreads) {
        (&s_tilemax[0][0])[e] = 0u;
        (&s_tilezsum[0][0])[e] = 0;
        (&s_tilezabs[0][0])[e] = 0;
    }
    if (tid < kMaxMem * kMaxM) (&s_tsum[0][0])[tid] = 0;
    __syncthreads();
    pdl_launch_dependents();

    auto block_of = [&](int b, int& l, int& rho) {
        const int g = a2 + b;
        l = member_of(P.t2_off, P.nmem, g);
        rho = g - P.t2_off[l];
    };

    if (warp == 0) {
        // ================================================================ producer
        if (lane == 0) {
            int i = 0;
            for (; i < n1 + n2; ++i) {
                if (s_abort) break;
                const int s = i % ns;
                if (i >= ns && !tc::mbar_wait(empty(s), ((i / ns) - 1) & 1, P.err)) {
                    s_abort = 1;
                    break;
                }
                if (i < n1) {
                    tc::mbar_arrive_expect_tx(full(s), static_cast<uint32_t>(64 * P.H1));
                    tc::tma_load_2d(slot_addr(s), &P.mem[s_tl[i]].tmV, kTileWords * s_tc[i], s_trb[i] * P.H1, full(s));
                } else {
                    int l, rho;
                    block_of(i - n1, l, rho);
                    const Member& m = P.mem[l];
                    tc::mbar_arrive_expect_tx(full(s), static_cast<uint32_t>(m.BW * m.R2 * 4));
                    tc::tma_load_2d(slot_addr(s), &m.tmU, 0, rho * m.R2, full(s));
                }
            }
            s_issued = i;
        }
    } else {
        // ================================================================ consumers
        const int cw = warp - 1;      // consumer warp 0..7
        const int ctid = tid - 32;    // consumer thread 0..255
        constexpr int kCT = 32 * kCW;
        uint2* const ztab = reinterpret_cast<uint2*>(gbase + P.off_ztab);   // [n1][KS][32]
        float* const zs = reinterpret_cast<float*>(gbase + P.off_zs);       // [n1][M][H1]
        uint16_t* const s2s = reinterpret_cast<uint16_t*>(gbase + P.off_s2s);  // [n1][H1]
        uint16_t* const s1s = reinterpret_cast<uint16_t*>(gbase + P.off_s1s);  // [n2][R2max]
        long long* const pbuf = reinterpret_cast<long long*>(gbase + P.off_dw) + cw * 64 * kMaxM;  // this warp's

        // ---- weights first (before the wait for the previous kernel): max |s2| of every member,
        // s2 of this CTA's stage-1 rows, s1 of its stage-2 rows, cleared digit tables
#pragma unroll 1
        for (int l = 0; l < P.nmem; ++l) {
            const uint16_t* s2 = P.mem[l].s2;
            uint32_t mx = 0u;  // max of |s2| as fp16 magnitude bits (order-preserving)
            const int nv = P.d_in / 8;
#pragma unroll 1
            for (int v = ctid; v < nv; v += kCT) {
                const uint4 q = __ldg(reinterpret_cast<const uint4*>(s2) + v);
                const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) mx = max(mx, max(w[h] & 0x7fffu, (w[h] >> 16) & 0x7fffu));
            }
#pragma unroll 1
            for (int j = nv * 8 + ctid; j < P.d_in; j += kCT) mx = max(mx, static_cast<uint32_t>(__ldg(s2 + j)) & 0x7fffu);
            mx = __reduce_max_sync(0xffffffffu, mx);
            if (lane == 0) atomicMax(&s_s2max[l], __float_as_uint(f16_bits_to_float(static_cast<uint16_t>(mx))));
        }
#pragma unroll 1
        for (int e = ctid; e < n1 * P.H1; e += kCT) {
            const int t = e / P.H1, i = e - t * P.H1;
            const int j = s_trb[t] * P.H1 + i;
            s2s[e] = (j < P.d_in) ? __ldg(P.mem[s_tl[t]].s2 + j) : static_cast<uint16_t>(0);
        }
#pragma unroll 1
        for (int e = ctid; e < n2 * P.R2max; e += kCT) {
            const int b = e / P.R2max, i = e - b * P.R2max;
            int l, rho;
            block_of(b, l, rho);
            const Member& m = P.mem[l];
            const int row = rho * m.R2 + i;
            s1s[e] = (i < m.R2 && row < m.d_out) ? __ldg(m.s1 + row) : static_cast<uint16_t>(0);
        }
        {
            uint4* z4 = reinterpret_cast<uint4*>(ztab);
            const int nz = n1 * KS * 16;
#pragma unroll 1
            for (int e = ctid; e < nz; e += kCT) z4[e] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
            for (int l = 0; l < P.nmem; ++l) {
                uint4* b4 = reinterpret_cast<uint4*>(gbase + P.mem[l].btab);
                const int nb = 8 * P.mem[l].ng * 16;
#pragma unroll 1
                for (int e = ctid; e < nb; e += kCT) b4[e] = make_uint4(0u, 0u, 0u, 0u);
            }
        }

        pdl_wait();  // x (and the workspace) may be written by the previous kernel
        // Launches on this workspace run in stream order and each adds G to the barrier counter,
        // which no CTA of this launch can move past a multiple of G before all have read it:
        // the launch index k = counter / G.  Launch k accumulates into zone half k & 1 and
        // clears the other half (last read by launch k - 1, complete) for launch k + 1.
        if (ctid == 0) s_launch = *reinterpret_cast<volatile unsigned long long*>(P.sync) / G;
        consumers_sync();
        const int parity = static_cast<int>(s_launch & 1ull);
        long long* const half = P.zone + parity * kZoneHalf;
        long long* const bounds = bounds_base + parity * (kMaxMem * kMaxM);
        {
            long long* other = P.zone + (parity ^ 1) * kZoneHalf;
            const int e0 = static_cast<int>(static_cast<long long>(kZoneHalf / 2) * cta / G);
            const int e1 = static_cast<int>(static_cast<long long>(kZoneHalf / 2) * (cta + 1) / G);
#pragma unroll 1
            for (int e = e0 + ctid; e < e1; e += kCT) reinterpret_cast<uint4*>(other)[e] = make_uint4(0u, 0u, 0u, 0u);
            if (cta == 0 && ctid < kMaxMem * kMaxM) bounds_base[(parity ^ 1) * (kMaxMem * kMaxM) + ctid] = 0;
        }

        // ---- max |x| per batch row over the whole input (bf16 magnitude bits order like the
        // values), and z of this CTA's stage-1 rows with each tile's maximum.  One pass issues
        // up to 16 loads of each kind per thread before it uses any.
        {
            constexpr int U = 8;
            const int lgH1 = __ffs(P.H1) - 1, lgM = M - 1;  // H1 a power of two, M 1 or 2
            uint32_t mx0 = 0u, mx1 = 0u;
            const int total = M * P.d_in;
            const int nv = total / 8;
            const int nz = n1 * M * P.H1;
            const int rounds = (max(nv, nz) + U * kCT - 1) / (U * kCT);
#pragma unroll 1
            for (int rd = 0; rd < rounds; ++rd) {
                uint4 xv[U];
                uint16_t xz[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = (rd * U + u) * kCT + ctid;
                    xv[u] = (v < nv) ? *reinterpret_cast<const uint4*>(P.x + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
                    const int tm = v >> lgH1, t = tm >> lgM, m = tm & lgM;
                    const int j = s_trb[min(t, kMaxTiles1 - 1)] * P.H1 + (v & (P.H1 - 1));
                    xz[u] = (v < nz && j < P.d_in) ? P.x[static_cast<int64_t>(m) * P.d_in + j] : static_cast<uint16_t>(0);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = (rd * U + u) * kCT + ctid;
                    // magnitudes of the eight bf16 values, two per word
                    const uint32_t a = __vmaxu2(__vmaxu2(xv[u].x & 0x7fff7fffu, xv[u].y & 0x7fff7fffu),
                                                __vmaxu2(xv[u].z & 0x7fff7fffu, xv[u].w & 0x7fff7fffu));
                    const uint32_t vm = max(a & 0xffffu, a >> 16);
                    if (8 * v + 8 <= P.d_in) {
                        mx0 = max(mx0, vm);
                    } else if (8 * v >= P.d_in) {
                        mx1 = max(mx1, vm);
                    } else {  // the vector that holds the end of row 0
                        const uint32_t w[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            const uint32_t b = (w[h >> 1] >> (16 * (h & 1))) & 0x7fffu;
                            if (8 * v + h < P.d_in) mx0 = max(mx0, b);
                            else mx1 = max(mx1, b);
                        }
                    }
                    if (v < nz) {
                        const int t = (v >> lgH1) >> lgM;
                        zs[v] = f16_bits_to_float(s2s[(t << lgH1) + (v & (P.H1 - 1))]) * bf16_bits_to_float(xz[u]);
                    }
                }
            }
#pragma unroll 1
            for (int e = nv * 8 + ctid; e < total; e += kCT) {
                const uint32_t a = static_cast<uint32_t>(P.x[e]) & 0x7fffu;
                if (e < P.d_in) mx0 = max(mx0, a);
                else mx1 = max(mx1, a);
            }
            mx0 = __reduce_max_sync(0xffffffffu, mx0);
            mx1 = __reduce_max_sync(0xffffffffu, mx1);
            if (lane == 0) {
                atomicMax(&s_xmax[0], __float_as_uint(bf16_bits_to_float(static_cast<uint16_t>(mx0))));
                if (M > 1) atomicMax(&s_xmax[1], __float_as_uint(bf16_bits_to_float(static_cast<uint16_t>(mx1))));
            }
        }
        consumers_sync();
        // each tile's maximum |z| (a warp per 32 values; H1 is a multiple of 32)
#pragma unroll 1
        for (int e0 = cw * 32; e0 < n1 * M * P.H1; e0 += kCT) {
            const int tm = e0 / P.H1;
            const int t = tm / M, m = tm - t * M;
            const uint32_t v = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(zs[e0 + lane])));
            if (lane == 0) atomicMax(&s_tilemax[t][m], v);
        }
        consumers_sync();
        // common exponent per member and batch row: Q = 16 + (22 - e(max|s2| max|x|))
        if (ctid < P.nmem * M) {
            const int l = ctid / M, m = ctid - l * M;
            const double bound = static_cast<double>(__uint_as_float(s_s2max[l])) * static_cast<double>(__uint_as_float(s_xmax[m]));
            const int e = static_cast<int>((__double_as_longlong(bound) >> 52) & 0x7ff) - 1022;
            s_Q[l][m] = (bound > 0.0) ? (22 - e) + 16 : 0;
        }
        consumers_sync();
        // each tile's run shift: from the run's maximum, at most Q
        if (ctid < n1 * M) {
            const int t = ctid / M, m = ctid - t * M;
            float v = 0.0f;
            for (int u = s_rfirst[t]; u <= s_rlast[t]; ++u) v = fmaxf(v, __uint_as_float(s_tilemax[u][m]));
            const int Q = s_Q[s_tl[t]][m];
            s_tilesh[t][m] = (v > 0.0f) ? min(22 - exp_of(v), Q) : Q;
        }
        consumers_sync();
        // ---- z's digit table: for tile t, K step kb and lane (gid, tig), .x holds digit
        // column gid of rows 32 kb + 4 tig + i (byte i), .y of rows 32 kb + 16 + 4 tig + i.
        // A task is (t, kb, tig, half); the 8 KS tasks of a tile are consecutive, so aligned
        // lane groups reduce each tile's sums of z_q and |z_q|.
        {
            const int tasks = n1 * KS * 8;
            const int gw = min(32, 8 * KS);
#pragma unroll 1
            for (int e0 = cw * 32; e0 < tasks; e0 += kCT) {
                const int e = e0 + lane;
                const bool on = e < tasks;
                const int half = e & 1, tg = (e >> 1) & 3, kt = e >> 3;  // kt = t KS + kb
                const int t = on ? kt / KS : 0, kb = kt - t * KS;
#pragma unroll
                for (int m = 0; m < kMaxM; ++m) {
                    long long qs = 0, qa = 0;
                    if (on && m < M) {
                        const double mul = pow2_d(s_tilesh[t][m]);
                        uint32_t d0 = 0u, d1 = 0u, d2 = 0u;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int jl = 32 * kb + 16 * half + 4 * tg + i;
                            const int qv = __double2int_rn(static_cast<double>(zs[(t * M + m) * P.H1 + jl]) * mul);
                            qs += qv;
                            qa += abs(qv);
                            uint32_t a0, a1, a2;
                            digits3(qv, a0, a1, a2);
                            d0 |= a0 << (8 * i);
                            d1 |= a1 << (8 * i);
                            d2 |= a2 << (8 * i);
                        }
                        uint32_t* zt = reinterpret_cast<uint32_t*>(ztab + kt * 32);
                        zt[2 * (4 * (3 * m + 0) + tg) + half] = d0;
                        zt[2 * (4 * (3 * m + 1) + tg) + half] = d1;
                        zt[2 * (4 * (3 * m + 2) + tg) + half] = d2;
                    }
                    if (m < M) {
                        qs = group_sum(qs, gw);
                        qa = group_sum(qa, gw);
                        if (on && (lane & (gw - 1)) == 0) {
                            atomicAdd(reinterpret_cast<unsigned long long*>(&s_tilezsum[t][m]), static_cast<unsigned long long>(qs));
                            atomicAdd(reinterpret_cast<unsigned long long*>(&s_tilezabs[t][m]), static_cast<unsigned long long>(qa));
                        }
                    }
                }
            }
        }
        consumers_sync();

        // ---- stage 1: MMAs over the tiles; exact partials of t into the accumulator per run
        {
            int acc[2][2][4];
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[a][b][e] = 0;
            const uint32_t msk = 0x01010101u << gid;
#pragma unroll 1
            for (int t = 0; t < n1; ++t) {
                const int l = s_tl[t], c = s_tc[t];
                const int s = t % ns;
                if (!tc::mbar_wait(full(s), (t / ns) & 1, P.err)) s_abort = 1;
                consumers_sync();
                if (s_abort) break;
                const uint32_t slot = slot_addr(s);
                // in-place transpose: thread (q, p), rows read in a rotated order
#pragma unroll 1
                for (int task = ctid; task < P.H1; task += kCT) {
                    const int q = task >> 2, p = task & 3;
                    // instruction i reads row 4q + ((i + (q & 1)) & 3); the transpose's last byte
                    // permutation puts the rows back in order
                    uint4 rw[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) rw[i] = lds128(s1_unit_addr(slot, 4 * q + ((i + (q & 1)) & 3), p));
                    const uint32_t sel_lo = (q & 1) ? 0x4105u : 0x5410u;
                    const uint32_t sel_hi = (q & 1) ? 0x6327u : 0x7632u;
                    uint32_t o[4][4];  // [a][b] : T[q][4p + a][b]
                    transpose_rows(rw[0].x, rw[1].x, rw[2].x, rw[3].x, sel_lo, sel_hi, o[0]);
                    transpose_rows(rw[0].y, rw[1].y, rw[2].y, rw[3].y, sel_lo, sel_hi, o[1]);
                    transpose_rows(rw[0].z, rw[1].z, rw[2].z, rw[3].z, sel_lo, sel_hi, o[2]);
                    transpose_rows(rw[0].w, rw[1].w, rw[2].w, rw[3].w, sel_lo, sel_hi, o[3]);
                    // T[q][4p + a] goes to row 4q + (a ^ (q & 3)), unit p
#pragma unroll
                    for (int a = 0; a < 4; ++a)
                        sts128(s1_unit_addr(slot, 4 * q + (a ^ (q & 3)), p), make_uint4(o[a][0], o[a][1], o[a][2], o[a][3]));
                }
                tc::fence_proxy_async_smem();
                consumers_sync();
                // this warp's two words of the chunk
                const Member& mb = P.mem[l];
                if (16 * c + 2 * cw < mb.nw) {
                    const uint2* zt = ztab + t * KS * 32;
#pragma unroll 1
                    for (int kb = 0; kb < KS; ++kb) {
                        const uint2 bz = zt[kb * 32 + lane];
#pragma unroll
                        for (int wi = 0; wi < 2; ++wi) {
                            const int w = 2 * cw + wi;
                            const uint4 T1 = lds128(s1_T_addr(slot, 8 * kb + tig, w));
                            const uint4 T2 = lds128(s1_T_addr(slot, 8 * kb + 4 + tig, w));
                            mma_u8s8(acc[wi][0], T1.x & msk, T1.y & msk, T2.x & msk, T2.y & msk, bz.x, bz.y);
                            mma_u8s8(acc[wi][1], T1.z & msk, T1.w & msk, T2.z & msk, T2.w & msk, bz.x, bz.y);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(empty(s));
                if (s_rlast[t] == t) {
                    // end of the run: its sums of z_q and |z_q|, then this warp's partials
                    long long zs0 = 0, zs1 = 0, za0 = 0, za1 = 0;
                    for (int u = s_rfirst[t]; u <= t; ++u) {
                        zs0 += s_tilezsum[u][0];
                        zs1 += s_tilezsum[u][1];
                        za0 += s_tilezabs[u][0];
                        za1 += s_tilezabs[u][1];
                    }
                    if (cw == 0 && lane < M) {
                        const long long b = (lane == 0 ? za0 : za1) << (s_Q[l][lane] - s_tilesh[t][lane]);
                        atomicAdd(reinterpret_cast<unsigned long long*>(bounds + l * kMaxM + lane), static_cast<unsigned long long>(b));
                    }
                    flush_run(mb, half, c, cw, lane, M, zs0, zs1, s_tilesh[t], s_Q[l], acc, pbuf);
                }
            }
        }

        // ---- grid barrier: every CTA's partials are in the accumulator.  The arrival is a
        // release reduction (it orders this CTA's partials, seen through the CTA barrier, before
        // it); launch k is complete when the counter reaches (k + 1) G.
        consumers_sync();
        if (ctid == 0) {
            asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(P.sync) : "memory");
            const unsigned long long target = (s_launch + 1) * static_cast<unsigned long long>(G);
            const uint64_t t0 = tc::globaltimer_ns();
            while (ld_acquire_u64(P.sync) < target) {
                if (tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) {
                    flag_error(P.err, kErrTimeout);
                    s_abort = 1;
                    break;
                }
            }
        }
        consumers_sync();

        // ---- stage 2 prologue: t of the members this CTA's blocks belong to, as 23-bit digits.
        // The shift comes from the exact bound sum |z_q| 2^(Q - shift) >= |t|, so one pass
        // suffices: a task is (word w, bit offset s, batch row m); it reads the four t of k =
        // 32 w + s + 8 i and writes whole words of the digit table.
        int l_lo = P.nmem, l_hi = -1;
        if (n2 > 0) {
            int rho;
            block_of(0, l_lo, rho);
            block_of(n2 - 1, l_hi, rho);
        }
        if (!s_abort) {
            int32_t* const tq = reinterpret_cast<int32_t*>(gbase + P.off_tq);  // [M][r] of the member in hand
#pragma unroll 1
            for (int l = l_lo; l <= l_hi; ++l) {
                const Member& mb = P.mem[l];
                const long long* tl = half + mb.tacc;
                // the bound and up to kTPer accumulator values per thread in one round of loads
                const int E = M * mb.r;
                const long long b0 = bounds[l * kMaxM];
                const long long b1 = (M > 1) ? bounds[l * kMaxM + 1] : 0ll;
                const int d0 = max(0, (64 - __clzll(b0)) - 22), d1 = max(0, (64 - __clzll(b1)) - 22);
                long long ts0 = 0, ts1 = 0;
#pragma unroll 1
                for (int e0 = 0; e0 < E; e0 += kTPer * kCT) {
                    long long v[kTPer];
#pragma unroll
                    for (int u = 0; u < kTPer; ++u) {
                        const int e = e0 + u * kCT + ctid;
                        const int m = (e >= mb.r) ? 1 : 0, k = e - m * mb.r;
                        v[u] = (e < E) ? tl[static_cast<int64_t>(m) * mb.rp + k] : 0ll;
                    }
#pragma unroll
                    for (int u = 0; u < kTPer; ++u) {
                        const int e = e0 + u * kCT + ctid;
                        if (e < E) {
                            const int m = (e >= mb.r) ? 1 : 0;
                            const int d = m ? d1 : d0;
                            long long q = v[u];
                            if (d > 0) {  // round to nearest, ties to even
                                const long long fl = q >> d;
                                const long long rem = q - (fl << d);
                                const long long hf = 1ll << (d - 1);
                                q = fl + ((rem > hf || (rem == hf && (fl & 1))) ? 1 : 0);
                            }
                            if (m) ts1 += q;
                            else ts0 += q;
                            tq[e] = static_cast<int32_t>(q);
                        }
                    }
                }
                if (ctid < M) s_td[l][ctid] = ctid ? d1 : d0;
                ts0 = group_sum(ts0, 32);
                ts1 = group_sum(ts1, 32);
                if (lane == 0) {
                    atomicAdd(reinterpret_cast<unsigned long long*>(&s_tsum[l][0]), static_cast<unsigned long long>(ts0));
                    if (M > 1) atomicAdd(reinterpret_cast<unsigned long long*>(&s_tsum[l][1]), static_cast<unsigned long long>(ts1));
                }
                consumers_sync();
                // digit table: a task is (word w, bit offset s, batch row m) and writes whole
                // words: byte i of column 3m + q holds digit q of t_q(32 w + s + 8 i)
                uint32_t* bt = reinterpret_cast<uint32_t*>(gbase + mb.btab);
                const int tasks = mb.nw * 8 * M;
#pragma unroll 1
                for (int e = ctid; e < tasks; e += kCT) {
                    const int m = (e >= mb.nw * 8) ? 1 : 0, ws_ = e - m * mb.nw * 8;
                    const int s_ = ws_ & 7, w = ws_ >> 3;
                    uint32_t W0 = 0u, W1 = 0u, W2 = 0u;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int k = 32 * w + s_ + 8 * i;
                        const int q = (k < mb.r) ? tq[m * mb.r + k] : 0;
                        uint32_t a0, a1, a2;
                        digits3(q, a0, a1, a2);
                        W0 |= a0 << (8 * i);
                        W1 |= a1 << (8 * i);
                        W2 |= a2 << (8 * i);
                    }
                    const int g = w >> 3, tg = (w & 7) >> 1, hf = w & 1;
                    uint32_t* dst = bt + 2 * ((s_ * mb.ng + g) * 32 + 12 * m + tg) + hf;
                    dst[0] = W0;
                    dst[8] = W1;   // column 3m + 1: four lanes on
                    dst[16] = W2;  // column 3m + 2
                }
                consumers_sync();
            }
        }
        consumers_sync();

        // ---- stage 2: all consumer warps work on each block.  For a pair of 16-row M-tiles,
        // the 8 ng (word group, bit offset) units are split evenly over the warps; each warp's
        // exact partial sums of P meet in shared memory.
        if (!s_abort) {
#pragma unroll 1
            for (int b = 0; b < n2; ++b) {
                const int i = n1 + b, s = i % ns;
                if (!tc::mbar_wait(full(s), (i / ns) & 1, P.err)) s_abort = 1;
                consumers_sync();
                if (s_abort) break;
                int l, rho;
                block_of(b, l, rho);
                const Member& mb = P.mem[l];
                const uint32_t slot = slot_addr(s);
                const uint32_t bt = base + static_cast<uint32_t>(mb.btab);
                const int ng = mb.ng, BW = mb.BW;
                const int u0 = (cw * 8 * ng) / kCW, u1 = ((cw + 1) * 8 * ng) / kCW;  // units g * 8 + s
#pragma unroll 1
                for (int pr = 0; pr < mb.R2 / 32; ++pr) {
                    const int row0 = rho * mb.R2 + 32 * pr;
                    if (row0 >= mb.d_out) break;
                    int acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
                    // rows gid and gid + 8 of M-tiles 0 and 1 of the pair
                    const uint32_t r00 = slot + static_cast<uint32_t>(((32 * pr + gid) * BW + 2 * tig) * 4);
                    const uint32_t r01 = r00 + static_cast<uint32_t>(8 * BW * 4);
                    const uint32_t r10 = r00 + static_cast<uint32_t>(16 * BW * 4);
                    const uint32_t r11 = r00 + static_cast<uint32_t>(24 * BW * 4);
                    int gcur = -1;
                    uint2 u00 = make_uint2(0u, 0u), u01 = u00, u10 = u00, u11 = u00;
#pragma unroll 1
                    for (int u = u0; u < u1; ++u) {
                        const int g = u >> 3, s_ = u & 7;
                        if (g != gcur) {
                            const uint32_t go = static_cast<uint32_t>(32 * g);
                            u00 = lds64(r00 + go);
                            u01 = lds64(r01 + go);
                            u10 = lds64(r10 + go);
                            u11 = lds64(r11 + go);
                            gcur = g;
                        }
                        // the A bytes of offset s hold bit s: shifted down, every offset shares one
                        // accumulator
                        const uint32_t m1 = 0x01010101u;
                        const uint2 bb = lds64(bt + static_cast<uint32_t>(((s_ * ng + g) * 32 + lane) * 8));
                        mma_u8s8(acc[0], (u00.x >> s_) & m1, (u01.x >> s_) & m1, (u00.y >> s_) & m1, (u01.y >> s_) & m1, bb.x, bb.y);
                        mma_u8s8(acc[1], (u10.x >> s_) & m1, (u11.x >> s_) & m1, (u10.y >> s_) & m1, (u11.y >> s_) & m1, bb.x, bb.y);
                    }
                    // this warp's partial P of each row, into its slice of the buffer
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int rh = 0; rh < 2; ++rh) {
                            long long P0, P1;
                            combine_cols(acc[mt][2 * rh], acc[mt][2 * rh + 1], tig, P0, P1);
                            const int rl = 16 * mt + 8 * rh + gid;
                            if (tig == 0) pbuf[2 * rl] = P0;
                            if (tig == 1) pbuf[2 * rl + 1] = P1;
                        }
                    consumers_sync();
                    if (ctid < 32 * M) {
                        // y = s1 (2 P - sum t_q) 2^(d - Q), rounded once to bf16
                        const int rl = ctid & 31, m = ctid >> 5, row = row0 + rl;
                        long long Pm = 0;
                        const long long* pall = reinterpret_cast<const long long*>(gbase + P.off_dw);
#pragma unroll
                        for (int w = 0; w < kCW; ++w) Pm += pall[w * 64 * kMaxM + 2 * rl + m];
                        if (row < mb.d_out) {
                            const double s1v = static_cast<double>(f16_bits_to_float(s1s[b * P.R2max + 32 * pr + rl]));
                            const long long val = 2 * Pm - s_tsum[l][m];
                            const double yv = s1v * static_cast<double>(val) * pow2_d(s_td[l][m] - s_Q[l][m]);
                            mb.y[static_cast<int64_t>(m) * mb.d_out + row] = __bfloat16_as_ushort(__double2bfloat16(yv));
                        }
                    }
                    consumers_sync();
                }
                if (ctid == 0) mbar_arrive_cnt(empty(s), kCW);
            }
        }
    }

    // ---- all threads: no TMA copy may still be writing this CTA's shared memory at exit
    __syncthreads();
    if (tid == 0) {
        const int issued = s_issued;
        for (int i = max(0, issued - ns); i < issued; ++i) tc::mbar_wait(full(i % ns), (i / ns) & 1, P.err);
    }
}

}  // namespace ds
}  // namespace nq

// ------------------------------------------------------------------------------ host side
#include <algorithm>
#include <atomic>

namespace {

using nq::ds::Params;

constexpr size_t kStreamSmemBudget = 220 * 1024;  // plus a few KB of static shared memory
constexpr size_t kZoneOffset = NQ_WS_SYNC_BYTES;  // the accumulator follows the counters

int64_t rup(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// Box width of a U row: the smallest multiple of 8 words >= nw that is 8 or 24 mod 32, so that
// the 64-bit A-fragment loads of four consecutive rows fall in distinct banks.
int box_width(int nw) {
    int bw = static_cast<int>(rup(nw, 8));
    while ((bw % 32) != 8 && (bw % 32) != 24) bw += 8;
    return bw;
}

bool encode_u32_map(CUtensorMap* map, const uint32_t* base, int64_t rows, int64_t nw, int64_t ld, int box_w,
                    int box_rows, bool swizzle64) {
    auto enc = nq_host::tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(nw), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 4)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_w), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
               swizzle64 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct StreamPlan {
    Params p;
    size_t smem;
    int grid;
};

// Fills the launch parameters; false when the layers are outside this kernel's reach (the
// caller then uses the two-kernel path).
bool plan_stream(const nq_lrb_layer* const* Ls, int n, const uint16_t* x, uint16_t* const* ys, int M, void* ws,
                 StreamPlan& sp) {
    if (n < 1 || n > nq::ds::kMaxMem || M < 1 || M > nq::ds::kMaxM) return false;
    const int G = nq_host::sm_count();
    Params& p = sp.p;
    p = Params{};
    p.nmem = n;
    p.M = M;
    p.d_in = static_cast<int>(Ls[0]->d_in);
    p.x = x;
    if (Ls[0]->d_in > (1 << 17)) return false;  // int32 stage-1 sums of a run stay exact
    // stage-1 tile height: the tallest that still gives every CTA two tiles or more
    int nch = 0;
    for (int l = 0; l < n; ++l) {
        const nq_lrb_layer* L = Ls[l];
        if (L->d_in != Ls[0]->d_in || (L->ldu % 4) != 0 || (L->ldv % 4) != 0) return false;
        if (L->d_out > (1 << 30)) return false;
        const int nw = static_cast<int>(L->r / 32);
        if (nw > 248) return false;  // one U row must fit a TMA box (<= 256 words)
        nch += (nw + nq::ds::kTileWords - 1) / nq::ds::kTileWords;
    }
    p.H1 = 64;
    for (int h : {256, 128}) {
        if (static_cast<int64_t>(nch) * ((Ls[0]->d_in + h - 1) / h) >= 2 * G) {
            p.H1 = h;
            break;
        }
    }
    p.nrb = static_cast<int>((Ls[0]->d_in + p.H1 - 1) / p.H1);
    int slot = 64 * p.H1;
    size_t zone = 0;
    for (int l = 0; l < n; ++l) {
        const int nw = static_cast<int>(Ls[l]->r / 32);
        slot = std::max(slot, 32 * box_width(nw) * 4);
    }
    slot = static_cast<int>(rup(std::max(slot, 16384), 1024));
    p.slot_bytes = slot;
    int t1 = 0, t2 = 0;
    long long b2 = 0;
    p.R2max = 0;
    for (int l = 0; l < n; ++l) {
        const nq_lrb_layer* L = Ls[l];
        nq::ds::Member& m = p.mem[l];
        m.d_out = static_cast<int>(L->d_out);
        m.r = static_cast<int>(L->r);
        m.nw = m.r / 32;
        m.ng = (m.nw + 7) / 8;
        m.BW = box_width(m.nw);
        m.R2 = std::min(256, (slot / (m.BW * 4)) / 32 * 32);
        m.R2 = static_cast<int>(std::min<int64_t>(m.R2, rup(L->d_out, 32)));
        m.rp = static_cast<int>(rup(m.r, 512));
        m.nchunks = (m.nw + nq::ds::kTileWords - 1) / nq::ds::kTileWords;
        m.s1 = L->s1;
        m.s2 = L->s2;
        m.y = ys[l];
        m.tacc = static_cast<int>(zone);
        zone += static_cast<size_t>(M) * m.rp;
        m.b2_bytes = static_cast<long long>(m.BW) * m.R2 * 4;
        if (!encode_u32_map(&m.tmV, L->V, L->d_in, m.nw, L->ldv, nq::ds::kTileWords, p.H1, true)) return false;
        if (!encode_u32_map(&m.tmU, L->U, L->d_out, m.nw, L->ldu, m.BW, m.R2, false)) return false;
        p.t1_off[l] = t1;
        t1 += m.nchunks * p.nrb;
        p.t2_off[l] = t2;
        p.b2_cum[l] = b2;
        const int nb = static_cast<int>((L->d_out + m.R2 - 1) / m.R2);
        t2 += nb;
        b2 += static_cast<long long>(nb) * m.b2_bytes;
        p.R2max = std::max(p.R2max, m.R2);
    }
    p.t1_off[n] = t1;
    p.t2_off[n] = t2;
    p.b2_cum[n] = b2;
    if (zone > static_cast<size_t>(nq::ds::kZoneHalf)) return false;
    p.zone = reinterpret_cast<long long*>(static_cast<char*>(ws) + kZoneOffset);
    p.sync = reinterpret_cast<unsigned long long*>(ws);
    p.err = nq_host::error_word();
    if (!p.err) return false;
    // per-CTA maxima of tiles and blocks (stage-2 blocks are split by bytes: allow for rounding)
    p.n1max = (t1 + G - 1) / G;
    if (p.n1max > nq::ds::kMaxTiles1) return false;
    {
        int mx = 0;
        for (int b = 0; b < G; ++b) {
            auto start = [&](int bb) {
                const long long target = (b2 * bb + G - 1) / G;
                for (int l = 0; l < n; ++l)
                    if (target < p.b2_cum[l + 1])
                        return p.t2_off[l] + static_cast<int>((target - p.b2_cum[l] + p.mem[l].b2_bytes - 1) /
                                                               p.mem[l].b2_bytes);
                return t2;
            };
            mx = std::max(mx, start(b + 1) - start(b));
        }
        p.n2max = mx;
    }
    // shared memory: ring | z digit table | z | s2 | s1 | t digit tables
    const int KS = p.H1 / 32;
    size_t off = 0;
    const size_t ring = static_cast<size_t>(slot);
    auto carve = [&](size_t bytes, size_t align) {
        off = (off + align - 1) / align * align;
        const size_t o = off;
        off += bytes;
        return static_cast<int>(o);
    };
    // reserve room for the ring later: compute the fixed part first (offsets relative to the
    // end of the ring, rebased below)
    size_t fixed = 0;
    {
        off = 0;
        p.off_ztab = carve(static_cast<size_t>(p.n1max) * KS * 32 * 8, 16);
        p.off_zs = carve(static_cast<size_t>(p.n1max) * M * p.H1 * 4, 16);
        p.off_s2s = carve(static_cast<size_t>(p.n1max) * p.H1 * 2, 16);
        p.off_s1s = carve(static_cast<size_t>(p.n2max) * p.R2max * 2, 16);
        for (int l = 0; l < n; ++l) p.mem[l].btab = carve(static_cast<size_t>(8) * p.mem[l].ng * 32 * 8, 16);
        p.off_dw = carve(static_cast<size_t>(nq::ds::kCW) * 64 * nq::ds::kMaxM * 8, 16);
        size_t tqb = 0;
        for (int l = 0; l < n; ++l) tqb = std::max(tqb, static_cast<size_t>(M) * p.mem[l].r * 4);
        p.off_tq = carve(tqb, 16);
        fixed = off;
    }
    const size_t slack = 1024;  // the kernel aligns the dynamic base to 1024 bytes
    if (fixed + 2 * ring + slack > kStreamSmemBudget) return false;
    int ns = static_cast<int>((kStreamSmemBudget - fixed - slack) / ring);
    ns = std::min(ns, nq::ds::kMaxSlots);
    p.ns = ns;
    const int rebase = ns * slot;
    p.off_ztab += rebase;
    p.off_zs += rebase;
    p.off_s2s += rebase;
    p.off_s1s += rebase;
    p.off_dw += rebase;
    p.off_tq += rebase;
    for (int l = 0; l < n; ++l) p.mem[l].btab += rebase;
    sp.smem = static_cast<size_t>(rebase) + fixed + slack;
    sp.grid = G;
    return true;
}

}  // namespace

// Launches the single-kernel decode path when the layers are within its reach; returns
// NQ_ERR_SHAPE without launching anything otherwise (the caller falls back).
nq_status nq_launch_decode_stream(const nq_lrb_layer* const* Ls, int n, const uint16_t* x, uint16_t* const* ys,
                                  int64_t M, void* ws, cudaStream_t stream, bool pdl) {
    StreamPlan sp;
    if (!plan_stream(Ls, n, x, ys, static_cast<int>(M), ws, sp)) return NQ_ERR_SHAPE;
    static std::atomic<bool> attr_done[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(nq::ds::decode_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kStreamSmemBudget)) != cudaSuccess)
            return NQ_ERR_LAUNCH;
        attr_done[dev].store(true, std::memory_order_release);
    }
    // the grid barrier needs every CTA resident at once: one CTA per SM must fit
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, nq::ds::decode_stream_kernel, nq::ds::kThreads,
                                                      sp.smem) != cudaSuccess ||
        per_sm < 1) {
        cudaGetLastError();
        return NQ_ERR_SHAPE;
    }
    void* args[] = {&sp.p};
    return nq_host::launch_pdl(reinterpret_cast<const void*>(nq::ds::decode_stream_kernel), dim3(sp.grid),
                               dim3(nq::ds::kThreads), sp.smem, stream, args, pdl) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_LAUNCH;
}
