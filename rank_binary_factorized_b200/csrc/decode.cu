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
// Both stages run on the integer tensor path (mma.sync m16n8k32, u8 x s8 -> s32): the
// packed bits, masked per bit offset, are the A operand as they are; the activations,
// quantised to 23-bit fixed point and split into three base-256 digits, are the B operand.
// Stage 1 is a split-d_in reduction over thread-block clusters (one cluster per chunk of 256
// outputs, one block per row slice of V) that sum their exact partials in distributed
// shared memory; its owner blocks hand t over already quantised, as stage 2's digit table.
// Stage 2 gives every block a run of 16-row tiles of U and copies that table into shared
// memory.  The two kernels chain by programmatic dependent launch: each reads its weights
// before it waits for the previous grid.
#include <cooperative_groups.h>

#include <algorithm>
#include <cstdlib>

#include "nq_common.cuh"

namespace nq {

// ------------------------------------------------------------------ shared helpers
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Asks the copy engine to bring [src, src + bytes) into L2 (no completion to wait for);
// src and bytes are multiples of 16.
__device__ __forceinline__ void l2_prefetch_bulk(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// The three balanced base-256 digits of a 23-bit signed integer v = a0 + 2^8 a1 + 2^16 a2,
// each in [-128, 127], returned as s8 bytes.
__device__ __forceinline__ void digits3(int v, uint32_t& d0, uint32_t& d1, uint32_t& d2) {
    const int a0 = (v << 24) >> 24;  // the low byte, sign-extended
    const int v1 = (v - a0) >> 8;    // exact: v - a0 is a multiple of 256
    const int a1 = (v1 << 24) >> 24;
    const int a2 = (v1 - a1) >> 8;
    d0 = static_cast<uint32_t>(a0) & 255u;
    d1 = static_cast<uint32_t>(a1) & 255u;
    d2 = static_cast<uint32_t>(a2) & 255u;
}

// Balanced base-256 digit q (0, 1, 2) of a 23-bit signed integer, as an s8 byte.
__device__ __forceinline__ uint32_t digit_byte(int v, int q) {
    int d0 = ((v + 128) & 255) - 128;
    if (q == 0) return static_cast<uint32_t>(d0) & 255u;
    int v1 = (v - d0) >> 8;
    int d1 = ((v1 + 128) & 255) - 128;
    if (q == 1) return static_cast<uint32_t>(d1) & 255u;
    return static_cast<uint32_t>((v1 - d1) >> 8) & 255u;
}


// Stage 2's B table (t's digits), which stage 1 writes.
// B table layout: the two B-fragment words of lane (gid, tig) for bit offset s, word group g
// (8 words) and column tile nt sit next to each other, lanes in order, so one 64-bit load per
// lane and MMA reads 256 contiguous bytes:
//   word ((((s * ng + g) * NT + nt) * 32 + 4 * gid + tig) * 2 + half)
// holds the digits of column 8 nt + gid for word 8 g + tig + 4 half.
template <int NT>
__device__ __forceinline__ int s2_bidx(int s_, int w, int col, int ng) {
    const int g = w >> 3, tg = w & 3, half = (w >> 2) & 1;
    return ((((s_ * ng + g) * NT + (col >> 3)) * 32 + 4 * (col & 7) + tg) * 2 + half);
}

// ------------------------------------------------------------------ stage 1 (integer MMA)
//
// t[m][k] = sum_j (2 v_jk - 1) z[m][j],  z = s2 (.) x,  v in {0, 1} the packed bits of V.
// V's bits run along k, the reduction runs along j, so four rows j..j+3 of one word column
// are first byte-transposed (8 PRMTs): word b of the result holds byte b of each of the four
// words.  For an output k with bit position g = k mod 8 in byte b = (k mod 32) / 8, the
// register  word_b & (0x01010101 << g)  holds the four bits v_{j..j+3,k} as the values
// {0, 2^g}: the A operand of mma.sync m16n8k32 (u8) for one row k and four K elements j.  z is
// quantised per CTA to 23-bit integers (three signed base-256 digits, the s8 B operand), so
// the products accumulate exactly in int32; each row's 2^g weight is shifted back exactly.
//
// Blocks form a thread-block cluster along d_in: block (c, q) owns word chunk c (8 words =
// 256 outputs k) and row slice q of V.  Each block turns its exact integer partial into an
// fp64 value with its own scale; after a cluster barrier, block q sums a 1/CS share of the
// chunk's outputs over the CS blocks' shared memory (distributed shared memory) in a fixed
// order and writes t.  No atomics, no global partials: deterministic.

// Threads per stage-1 block: 256 (one warp per word column) or 512 (two warps per word column,
// each half of the K range).  512 hides more latency on long row slices but fills the
// register file, so the block can no longer share an SM with the previous kernel's blocks
// under programmatic dependent launch; the host picks 512 only for long slices and NT <= 2.
constexpr int kS1Words = 8;            // words (of 32 outputs) per cluster chunk
constexpr int kS1Outs = kS1Words * 32;  // outputs k per chunk
constexpr int kS1PartCap = kS1Outs + 16;  // inbox doubles per batch row: ceil(256 / CS) CS <= 271

struct S1Params {
    const uint32_t* V;
    int64_t ldv;
    const uint16_t* s2;
    const uint16_t* x;
    float* t;
    int M;
    int64_t d_in;
    int r, nw;
    int rows_per_slice;  // rows of V per block (multiple of 32)
    int jc_rows;         // rows staged per pass (multiple of 32)
    int zstage;          // z of the slice (M x rows_per_slice fp32) is kept in shared memory
    // Stage 2's input, when tab != nullptr (otherwise t is written in fp32): t quantised with
    // one shift per batch row taken from a bound on |t| (sum over the slices of 2^-shift
    // sum_j |z_q|, the same in every cluster), as the digit table in s2_bidx layout; the
    // owner blocks' sums of t_q, tsum[(chunk * CS + rank) * M + m]; the shift, tsh[m].
    uint32_t* tab;
    long long* tsum;
    int* tsh;
    int nwp;  // words per row padded to a multiple of 8 (the table's geometry)
    int prefetch;  // prefetch the slice's rows of V into L2 (whole rows) before gathering strips
};

// Up to kMaxGroup projections that share their input x are launched as one grid: block
// column c belongs to member l when chunk_off[l] <= c < chunk_off[l + 1].
constexpr int kMaxGroup = NQ_MAX_GROUP;
struct S1Group {
    S1Params p[kMaxGroup];
    int chunk_off[kMaxGroup + 1];
    int n;
};

template <int NT>
struct S1Layout {
    static constexpr int SWZ = (NT == 1) ? 8 : 24;  // words per quad row of the z table
};

// 4x4 byte transpose: out[b] = (byte b of w0, byte b of w1, byte b of w2, byte b of w3)
__device__ __forceinline__ void byte_transpose4(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, uint32_t (&o)[4]) {
    const uint32_t t0 = __byte_perm(w0, w1, 0x5140);  // w0.b0 w1.b0 w0.b1 w1.b1
    const uint32_t t1 = __byte_perm(w0, w1, 0x7362);  // w0.b2 w1.b2 w0.b3 w1.b3
    const uint32_t t2 = __byte_perm(w2, w3, 0x5140);
    const uint32_t t3 = __byte_perm(w2, w3, 0x7362);
    o[0] = __byte_perm(t0, t2, 0x5410);
    o[1] = __byte_perm(t0, t2, 0x7632);
    o[2] = __byte_perm(t1, t3, 0x5410);
    o[3] = __byte_perm(t1, t3, 0x7632);
}

// 2^e as a double, written into the exponent field (|e| <= 1022)
__device__ __forceinline__ double pow2_d(int e) { return __longlong_as_double(static_cast<long long>(1023 + e) << 52); }

// Shift for a bound L >= 0 on |t|: with L < 2^e, |t * 2^(22 - e)| < 2^22.  The exponent comes
// from the bits of L, which is a normal double here (a positive L is at least 2^-126).
__device__ __forceinline__ int shift_for_bound(double L) {
    if (!(L > 0.0)) return 0;
    const int biased = static_cast<int>((__double_as_longlong(L) >> 52) & 0x7ff);
    const int e = biased - 1022;  // L = f 2^e with 0.5 <= f < 1
    return min(max(22 - e, -126), 126);
}

// GN: 1 for a single layer (member 0, resolved at compile time), kMaxGroup for a group.
template <int NT, int TH, int GN>
__global__ void __launch_bounds__(TH, 1) decode_stage1_kernel(const __grid_constant__ S1Group grp) {
    constexpr int kS1Threads = TH;
    constexpr int kKSplit = kS1Threads / (32 * kS1Words);  // warps per word column
    namespace cg = cooperative_groups;
    constexpr int SWZ = S1Layout<NT>::SWZ;
    extern __shared__ __align__(16) uint32_t smem1[];
    int li = 0;  // the member of the group this block works for
    if (GN > 1)
        while (li + 1 < grp.n && static_cast<int>(blockIdx.x) >= grp.chunk_off[li + 1]) ++li;
    const S1Params& p = grp.p[li];
    const int chunk = blockIdx.x - grp.chunk_off[li];
    const int nq_rows = p.jc_rows / 4;  // quads per pass
    const int nkb = p.jc_rows / 32;     // K steps per pass
    uint32_t* aws = smem1;                          // [8 words][nkb][2][4][4]
    uint32_t* zq = aws + kS1Words * (nkb * 32 + 4);  // [nq_rows][SWZ]
    int* red = reinterpret_cast<int*>(zq + nq_rows * SWZ);               // [256][NT*8]
    double* part = reinterpret_cast<double*>(red + kS1Outs * NT * 8);   // inbox [M][per][CS]
    float* zs_s = reinterpret_cast<float*>(part + p.M * (kS1PartCap + 16));  // [M][zld] when p.zstage
    const int zld = p.rows_per_slice + p.rows_per_slice / 32;             // one pad word per 32
    __shared__ float s_mul[NQ_MATVEC_MAX_M];
    __shared__ double s_dinv[NQ_MATVEC_MAX_M];  // 2^-shift: turns the exact integers into values
    __shared__ unsigned long long s_zsum[NQ_MATVEC_MAX_M];
    __shared__ unsigned long long s_zabs[NQ_MATVEC_MAX_M];  // sum_j |z_q| of the slice
    __shared__ long long s_tqsum[NQ_MATVEC_MAX_M];          // owner's sum of t_q
    __shared__ float s_wmax[kS1Threads / 32][NQ_MATVEC_MAX_M];

    cg::cluster_group cluster = cg::this_cluster();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;

    const int q = blockIdx.y;  // slice index == rank in the cluster
    const int CS = gridDim.y;
    const int64_t j0 = static_cast<int64_t>(q) * p.rows_per_slice;
    const int64_t j1 = min(p.d_in, j0 + p.rows_per_slice);
    const int wglob0 = chunk * kS1Words;

    // byte-transposed V quads of rows [jb, jb + jc_rows) into aws
    auto build_aws = [&](int64_t jb) {
        constexpr int U = 4;  // quads per thread in flight at once
        const int tasks = kS1Words * nq_rows;
        for (int e0 = tid; e0 < tasks; e0 += U * kS1Threads) {
            uint32_t v[U][4];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int e = e0 + u * kS1Threads;
                const int w = e % kS1Words, jq = e / kS1Words;
                const int wg = wglob0 + w;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int64_t j = jb + 4 * jq + i;
                    v[u][i] = (e < tasks && wg < p.nw && j < j1) ? __ldg(p.V + j * p.ldv + wg) : 0u;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int e = e0 + u * kS1Threads;
                if (e >= tasks) break;
                const int w = e % kS1Words, jq = e / kS1Words;
                uint32_t o[4];
                byte_transpose4(v[u][0], v[u][1], v[u][2], v[u][3], o);
                const int kb = jq >> 3, jl = jq & 7, t4 = jl & 3, half = jl >> 2;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int h = b >> 1, slot = (b & 1) + 2 * half;
                    aws[w * (nkb * 32 + 4) + ((kb * 2 + h) * 4 + t4) * 4 + slot] = o[b];
                }
            }
        }
    };

    // s2 of the slice (a weight) is read before the wait, into registers when the slice has
    // at most kS2Reg rows per thread
    constexpr int kS2Reg = 8;
    const bool s2reg = (j1 - j0) <= static_cast<int64_t>(kS2Reg) * kS1Threads;
    float s2r[kS2Reg];
#pragma unroll
    for (int i = 0; i < kS2Reg; ++i) {
        const int64_t j = j0 + tid + static_cast<int64_t>(i) * kS1Threads;
        s2r[i] = (s2reg && j < j1) ? f16_bits_to_float(__ldg(p.s2 + j)) : 0.0f;
    }
    if (warp == 0 && p.prefetch) {
        // the slice's rows of V, whole rows, split among the blocks of this row slice: one
        // contiguous range per block, prefetched into L2 by the copy engine, so that DRAM
        // streams full lines while the blocks' 32-byte strips are gathered from L2
        const int nc = grp.chunk_off[li + 1] - grp.chunk_off[li];
        const int64_t rows = j1 - j0;
        const int64_t r0 = j0 + (rows * chunk) / nc, r1 = j0 + (rows * (chunk + 1)) / nc;
        if (r1 > r0) {
            // from the 16-byte boundary at or below row r0 (V itself is 16-byte aligned) to the
            // last row's r/32-th word, rounded up to 16 bytes
            const uintptr_t b0 = reinterpret_cast<uintptr_t>(p.V + r0 * p.ldv);
            const uintptr_t b1 = reinterpret_cast<uintptr_t>(p.V + (r1 - 1) * p.ldv + p.nw);
            const char* a = reinterpret_cast<const char*>(b0 & ~static_cast<uintptr_t>(15));
            const int64_t units = static_cast<int64_t>((b1 - (b0 & ~static_cast<uintptr_t>(15)) + 15) / 16);
            constexpr int64_t kPiece = 2048;  // 16-byte units per prefetch (32 KB)
            for (int64_t u = static_cast<int64_t>(lane) * kPiece; u < units; u += 32 * kPiece)
                l2_prefetch_bulk(a + 16 * u, static_cast<uint32_t>(16 * min(kPiece, units - u)));
        }
    }
    build_aws(j0);  // weights only: may overlap the previous grid
    pdl_launch_dependents();
    pdl_wait();     // x may be written by the previous grid

    // ---- slice scale: |z_q| < 2^22, z_q = rint(z * 2^shift).  The batch rows are the inner,
    // unrolled loop, so every row's loads of x are in flight together.
    constexpr int MGS = (NT * 8 + 2) / 3;  // batch rows the B columns can hold (>= M)
    {
        float vmax[MGS];
#pragma unroll
        for (int m = 0; m < MGS; ++m) vmax[m] = 0.0f;
        if (s2reg && p.M == 1) {
#pragma unroll
            for (int i = 0; i < kS2Reg; ++i) {
                const int64_t j = j0 + tid + static_cast<int64_t>(i) * kS1Threads;
                if (j < j1) {
                    const float z = s2r[i] * bf16_bits_to_float(p.x[j]);
                    if (p.zstage) {
                        const int jl = static_cast<int>(j - j0);
                        zs_s[jl + (jl >> 5)] = z;
                    }
                    vmax[0] = fmaxf(vmax[0], fabsf(z));
                }
            }
        } else if (s2reg) {
#pragma unroll
            for (int i = 0; i < kS2Reg; ++i) {
                const int64_t j = j0 + tid + static_cast<int64_t>(i) * kS1Threads;
                if (j < j1) {
#pragma unroll
                    for (int m = 0; m < MGS; ++m) {
                        if (m < p.M) {
                            const float z = s2r[i] * bf16_bits_to_float(p.x[static_cast<int64_t>(m) * p.d_in + j]);
                            if (p.zstage) {
                                const int jl = static_cast<int>(j - j0);
                                zs_s[m * zld + jl + (jl >> 5)] = z;
                            }
                            vmax[m] = fmaxf(vmax[m], fabsf(z));
                        }
                    }
                }
            }
        } else {
#pragma unroll 4
            for (int64_t j = j0 + tid; j < j1; j += kS1Threads) {
                const float s2v = f16_bits_to_float(p.s2[j]);
#pragma unroll
                for (int m = 0; m < MGS; ++m) {
                    if (m < p.M) {
                        const float z = s2v * bf16_bits_to_float(p.x[static_cast<int64_t>(m) * p.d_in + j]);
                        if (p.zstage) {
                            const int jl = static_cast<int>(j - j0);
                            zs_s[m * zld + jl + (jl >> 5)] = z;
                        }
                        vmax[m] = fmaxf(vmax[m], fabsf(z));
                    }
                }
            }
        }
#pragma unroll
        for (int m = 0; m < MGS; ++m) {
            if (m < p.M) {
                float v = vmax[m];
                for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
                if (lane == 0) s_wmax[warp][m] = v;
            }
        }
        if (kKSplit > 1)  // several warps add into one output; otherwise each stores its own
            for (int e = tid; e < kS1Outs * NT * 8; e += kS1Threads) red[e] = 0;
        if (tid < NQ_MATVEC_MAX_M) {
            s_zsum[tid] = 0ull;
            s_zabs[tid] = 0ull;
            s_tqsum[tid] = 0ll;
        }
        __syncthreads();
        if (tid < p.M) {
            float v = 0.0f;
            for (int w = 0; w < kS1Threads / 32; ++w) v = fmaxf(v, s_wmax[w][tid]);
            int e = 0;
            frexpf(v, &e);
            const int sh = (v > 0.0f) ? min(max(22 - e, -126), 126) : 0;
            s_mul[tid] = ldexpf(1.0f, sh);
            s_dinv[tid] = ldexp(1.0, -sh);
        }
        __syncthreads();
    }
    // per-thread partial sums of the quantised z, per batch row (column group of the z table)
    constexpr int MG = (NT * 8 + 2) / 3;
    long long zacc[MG], zabs[MG];
#pragma unroll
    for (int m = 0; m < MG; ++m) zacc[m] = zabs[m] = 0;

    // ---- passes over the slice: z table, then MMAs; integer accumulators live in registers
    // two accumulator sets, even and odd K steps, for two independent MMA chains per tile
    int acc[2][2][NT][4];
#pragma unroll
    for (int par = 0; par < 2; ++par)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[par][h][nt][e] = 0;
    const int wcol = warp % kS1Words;          // word column of this warp
    const int khalf = warp / kS1Words;         // which share of the K steps
    const bool warp_active = (wglob0 + wcol) < p.nw;
    const uint32_t msk = 0x01010101u << gid;

    for (int64_t jb = j0; jb < j1; jb += p.jc_rows) {
        if (jb != j0) {
            __syncthreads();  // previous pass done with aws / zq
            build_aws(jb);
        }
        // z table: word zq[jq * SWZ + 3m + q] holds digit q of z_q(m, row jb + 4jq + i) in byte i;
        // one thread builds the three digit words of one (jq, m) from four z values.  Every row
        // of the pass lies in exactly one quad, so the quads' integers also give sum_j z_q(m, j).
        {
            const int64_t jend = min(j1, jb + p.jc_rows);
            for (int e = tid; e < nq_rows * MG; e += kS1Threads) {
                const int m = e % MG, jq = e / MG;  // MG is a compile-time constant
                uint32_t d0 = 0u, d1 = 0u, d2 = 0u;
                if (m < p.M) {
                    const float mul = s_mul[m];
                    const uint16_t* xm = p.x + static_cast<int64_t>(m) * p.d_in;
                    float zv[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int64_t j = jb + 4 * jq + i;
                        zv[i] = 0.0f;
                        if (j < jend) {
                            const int jl = static_cast<int>(j - j0);
                            zv[i] = p.zstage ? zs_s[m * zld + jl + (jl >> 5)]
                                             : f16_bits_to_float(p.s2[j]) * bf16_bits_to_float(xm[j]);
                        }
                    }
                    int qsum = 0, qabs = 0;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint32_t a0, a1, a2;
                        const int qv = __float2int_rn(zv[i] * mul);
                        qsum += qv;
                        qabs += abs(qv);
                        digits3(qv, a0, a1, a2);
                        d0 |= a0 << (8 * i);
                        d1 |= a1 << (8 * i);
                        d2 |= a2 << (8 * i);
                    }
#pragma unroll
                    for (int mm = 0; mm < MG; ++mm)
                        if (mm == m) {
                            zacc[mm] += qsum;
                            zabs[mm] += qabs;
                        }
                }
                uint32_t* dst = zq + jq * SWZ + 3 * m;
                if (m < p.M) {  // rows >= M: their D columns are never read
                    dst[0] = d0;
                    dst[1] = d1;
                    dst[2] = d2;
                }
            }
        }
        __syncthreads();

        if (warp_active) {
            const int w = wcol;
            const int kb_lo = (khalf * nkb) / kKSplit, kb_hi = ((khalf + 1) * nkb) / kKSplit;
            // operands of K step kb: the A words of both 16-output halves and the B digits;
            // the next step's are loaded from shared memory while this step's MMAs issue
            const uint32_t* abase = aws + w * (nkb * 32 + 4) + tig * 4;
            const uint32_t* zbase = zq + tig * SWZ + gid;
            struct Ops {
                uint4 a[2];
                uint32_t b[NT][2];
            };
            auto fetch = [&](int kb, Ops& o) {
#pragma unroll
                for (int h = 0; h < 2; ++h) o.a[h] = *reinterpret_cast<const uint4*>(abase + (kb * 2 + h) * 16);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    o.b[nt][0] = zbase[(8 * kb) * SWZ + nt * 8];
                    o.b[nt][1] = zbase[(8 * kb + 4) * SWZ + nt * 8];
                }
            };
            auto issue = [&](const Ops& o, int (&ac)[2][NT][4]) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_u8s8(ac[h][nt], o.a[h].x & msk, o.a[h].y & msk, o.a[h].z & msk, o.a[h].w & msk, o.b[nt][0],
                                 o.b[nt][1]);
            };
            Ops cur, nxt;
            if (kb_lo < kb_hi) fetch(kb_lo, cur);
            // two accumulator sets, even and odd K steps, for two independent MMA chains per tile
            for (int kb = kb_lo; kb < kb_hi; kb += 2) {
                if (kb + 1 < kb_hi) fetch(kb + 1, nxt);
                issue(cur, acc[0]);
                if (kb + 1 < kb_hi) {
                    if (kb + 2 < kb_hi) fetch(kb + 2, cur);
                    issue(nxt, acc[1]);
                }
            }
        }
    }

    // per-warp partial sums into s_zsum; read after the barriers of the reduction below
#pragma unroll
    for (int m = 0; m < MG; ++m) {
        if (m < p.M) {
            long long v = zacc[m], va = zabs[m];
            for (int off = 16; off > 0; off >>= 1) {
                v += __shfl_xor_sync(0xffffffffu, v, off);
                va += __shfl_xor_sync(0xffffffffu, va, off);
            }
            if (lane == 0) {
                atomicAdd(&s_zsum[m], static_cast<unsigned long long>(v));
                atomicAdd(&s_zabs[m], static_cast<unsigned long long>(va));
            }
        }
    }

    // ---- exact per-output integers: row gid of M-tile (w, h) is k = 32w + 8(2h) + gid,
    // row gid+8 is k = 32w + 8(2h+1) + gid; both carry the weight 2^gid
    if (warp_active) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int kl = 32 * wcol + 8 * (2 * h + (e >> 1)) + gid;
                    const int col = nt * 8 + 2 * tig + (e & 1);
                    const int v = (acc[0][h][nt][e] >> gid) + (acc[1][h][nt][e] >> gid);
                    if (kKSplit == 1) red[kl * (NT * 8) + col] = v;
                    else atomicAdd(&red[kl * (NT * 8) + col], v);
                }
    }
    __syncthreads();
    // ---- cluster reduction over the CS row slices.  Output k of the chunk belongs to the
    // block of rank k / per; every block stores its fp64 partial for k into slot [rank of
    // the sender] of the owner's inbox (distributed shared memory), one cluster barrier
    // publishes the stores, and each owner sums its slots in a fixed order.
    // The share per owner is ceil(256 / CS) outputs (the last owner's may run short); the
    // exact integer times the power of two 2^-shift is exact in fp64.
    const int per = (kS1Outs + CS - 1) / CS;
    // a power-of-two CS (the usual case) splits by shifts: no division on this critical path
    const bool per_pow2 = (CS & (CS - 1)) == 0;
    const int lg_per = per_pow2 ? 8 - (31 - __clz(CS)) : 0;
    for (int e = tid; e < p.M * kS1Outs; e += kS1Threads) {
        const int m = e / kS1Outs, kl = e - m * kS1Outs;
        const int* rr = red + kl * (NT * 8) + 3 * m;
        const long long P = static_cast<long long>(rr[0]) + (static_cast<long long>(rr[1]) << 8) +
                            (static_cast<long long>(rr[2]) << 16);
        const long long val = 2 * P - static_cast<long long>(s_zsum[m]);
        const int owner = per_pow2 ? (kl >> lg_per) : kl / per, ko = kl - owner * per;
        double* dst = cluster.map_shared_rank(part, owner);
        dst[(m * per + ko) * CS + q] = static_cast<double>(val) * s_dinv[m];
    }
    // the slice's bound on its share of |t| (exact), into every owner's inbox after the partials
    double* bound = part + p.M * kS1PartCap;  // [M][CS]
    if (p.tab)
        for (int e = tid; e < p.M * CS; e += kS1Threads) {
            const int m = e / CS, owner = e - m * CS;
            cluster.map_shared_rank(bound, owner)[m * CS + q] = static_cast<double>(s_zabs[m]) * s_dinv[m];
        }
    cluster.sync();
    // one shift per batch row for t: |t| <= L = the sum over the slices, taken as a fixed
    // pairwise tree over 16 leaves (ranks past CS are zeros, which add exactly), so L is the
    // same value in every thread, block and cluster, and |t_q| <= 2^22
    auto t_shift = [&](int m) {
        double v[16];
#pragma unroll
        for (int rank = 0; rank < 16; ++rank) v[rank] = (rank < CS) ? bound[m * CS + rank] : 0.0;
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
            for (int i = 0; i < w; ++i) v[i] = v[i] + v[i + w];
        return shift_for_bound(v[0]);
    };
    if (p.tab && chunk == 0 && q == 0 && tid < p.M) p.tsh[tid] = t_shift(tid);
    {
        // owner q: its `per` outputs, each the sum of the CS slices' partials in a fixed order
        // (four interleaved accumulators, then pairwise): a short dependent chain, few registers
        const int k_lo = q * per;
        const int ngp = p.nwp / 8;
        long long tqacc[MG];  // this thread's sum of t_q per batch row
#pragma unroll
        for (int m = 0; m < MG; ++m) tqacc[m] = 0;
        for (int e = tid; e < p.M * per; e += kS1Threads) {
            const int m = per_pow2 ? (e >> lg_per) : e / per, ko = e - m * per;
            if (k_lo + ko >= kS1Outs) continue;  // past the chunk: the last owner's share runs short
            const int64_t k = static_cast<int64_t>(wglob0) * 32 + k_lo + ko;
            double sum = 0.0;
            if (k < p.r) {
                const double* src = part + (m * per + ko) * CS;
                double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
                for (int rank = 0; rank < CS; rank += 4) {
                    a0 += src[rank];
                    if (rank + 1 < CS) a1 += src[rank + 1];
                    if (rank + 2 < CS) a2 += src[rank + 2];
                    if (rank + 3 < CS) a3 += src[rank + 3];
                }
                sum = (a0 + a1) + (a2 + a3);
            }
            if (p.tab) {
                // t_q's three digits, byte (k / 8) % 4 of the table words for (k % 8, k / 32);
                // outputs past r (up to the padded word count) get zero digits
                const int tq = (k < p.r) ? __double2int_rn(sum * pow2_d(t_shift(m))) : 0;
#pragma unroll
                for (int mm = 0; mm < MG; ++mm)
                    if (mm == m) tqacc[mm] += tq;
                uint32_t d0, d1, d2;
                digits3(tq, d0, d1, d2);
                const int w = static_cast<int>(k >> 5), s_ = static_cast<int>(k & 7), b = static_cast<int>((k >> 3) & 3);
                uint8_t* tb = reinterpret_cast<uint8_t*>(p.tab);
                tb[4 * s2_bidx<NT>(s_, w, 3 * m, ngp) + b] = static_cast<uint8_t>(d0);
                tb[4 * s2_bidx<NT>(s_, w, 3 * m + 1, ngp) + b] = static_cast<uint8_t>(d1);
                tb[4 * s2_bidx<NT>(s_, w, 3 * m + 2, ngp) + b] = static_cast<uint8_t>(d2);
            } else if (k < p.r) {
                p.t[static_cast<int64_t>(m) * p.r + k] = static_cast<float>(sum);
            }
        }
        if (p.tab) {
            // the block's sum of t_q per batch row: warp sums, then one shared add per warp
#pragma unroll
            for (int m = 0; m < MG; ++m) {
                if (m < p.M) {
                    long long v = tqacc[m];
                    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                    if (lane == 0 && v != 0)
                        atomicAdd(reinterpret_cast<unsigned long long*>(&s_tqsum[m]), static_cast<unsigned long long>(v));
                }
            }
            __syncthreads();
            if (tid < p.M) p.tsum[(static_cast<int64_t>(chunk) * CS + q) * p.M + tid] = s_tqsum[tid];
        }
    }
}

// ------------------------------------------------------------------ stage 2 (integer MMA)
//
// y[m][i] = s1_i * sum_k (2 u_ik - 1) t[m][k] with u in {0, 1} the packed bits of U.
// Stage 1 quantises t per batch row to a 23-bit fixed-point integer t_q = rint(t * 2^sh)
// (|t_q| <= 2^22, sh from a bound on |t|), split into three signed base-256 digits (planes)
// t_q = d0 + 2^8 d1 + 2^16 d2, and writes them as this kernel's B table.
// The packed words feed mma.sync m16n8k32 (A u8, B s8, D s32) directly: for a bit offset
// s in 0..7 the register  word & (0x01010101 << s)  holds, in its four bytes, the bits
// s, s+8, s+16, s+24 of the word as the values {0, 2^s} -- four K elements for one AND.
// The B operand supplies the t digits for those same four k, so the MMA for offset s
// accumulates 2^s * sum u_ik d_q(k) over k = s (mod 8); separate accumulators per s are
// shifted back (exactly: each is a multiple of 2^s) and summed.  Everything up to the final
// scale is integer arithmetic, so the result is exact for the quantised t and independent of
// summation order.
// Threads per stage-2 block: 256, or 512 for many M-tiles per block at NT = 1 (see stage 1).

struct S2Params {
    const uint32_t* U;
    int64_t ldu;
    const uint16_t* s1;
    // t as stage 1 leaves it: the digit table (s2_bidx layout, 8 nwp NT 8 words), the owner
    // blocks' sums of t_q (tsum_n per batch row, [i][M]) and the shift per batch row
    const uint32_t* tab;
    const long long* tsum;
    int tsum_n;
    const int* tsh;
    uint16_t* y;
    int M;
    int64_t d_out;
    int r, nw, nwp;      // rank, words per row, words padded to a multiple of 8
    int su;              // shared-memory row stride of U (words), = 4 (mod 32)
    int mt_total;        // 16-row M-tiles of U
    int chunk_mt;        // M-tiles staged in shared memory at a time
    // gradient mode (grad != nullptr): instead of y, grad[i] = sum_m cot[m][i] (U t_m)_i, the
    // derivative of sum_m <cot_m, y_m> with respect to s1_i; cot [M][d_out] bf16, grad fp32
    const uint16_t* cot;
    float* grad;
};

// Stage-2 blocks [cta_off[l], cta_off[l + 1]) work for member l of the group.  In the paired
// form (gate and up of an MLP block, equal d_out) every block works for both members on the
// same rows and writes h = bf16(silu(bf16(gate)) * bf16(up)) to member 0's y.
struct S2Group {
    S2Params p[kMaxGroup];
    int cta_off[kMaxGroup + 1];
    int n;
};

// h from the bf16 gate and up values: the same function as the elementwise SiLU.mul kernel
__device__ __forceinline__ uint16_t silu_mul_bf16(uint16_t g, uint16_t u) {
    const float gf = bf16_bits_to_float(g);
    const float sg = gf / (1.0f + expf(-gf));
    return float_to_bf16_bits(sg * bf16_bits_to_float(u));
}

// One member's share of stage 2 in shared memory: its digit table, the staged rows of U, the
// per-row integer sums and the staged s1.
struct S2Smem {
    uint32_t* bt;    // 8 * nwp * NT*8 words (s2_bidx)
    uint32_t* ublk;  // [chunk_mt*16][su]
    int* red;        // [chunk_mt*16][NT*8]
    float* s1_s;     // [chunk_mt*16]
};

template <int NT>
__device__ __forceinline__ size_t s2_smem_words(const S2Params& p) {
    return static_cast<size_t>(8) * p.nwp * NT * 8 + static_cast<size_t>(p.chunk_mt) * 16 * p.su +
           static_cast<size_t>(p.chunk_mt) * 16 * NT * 8 + static_cast<size_t>(p.chunk_mt) * 16;
}

template <int NT>
__device__ __forceinline__ S2Smem s2_carve(const S2Params& p, uint32_t* base) {
    S2Smem m;
    m.bt = base;
    m.ublk = m.bt + 8 * p.nwp * NT * 8;
    m.red = reinterpret_cast<int*>(m.ublk + p.chunk_mt * 16 * p.su);
    m.s1_s = reinterpret_cast<float*>(m.red + p.chunk_mt * 16 * NT * 8);
    return m;
}

// The MMAs of M-tiles [c0, c0 + nmt) of one member (rows staged in sm.ublk), added into sm.red:
// each warp takes an equal, contiguous share of the (M-tile, word-group) pairs in M-tile-major
// order and flushes its accumulators whenever its run leaves an M-tile.
template <int NT, int kWarps>
__device__ __forceinline__ void s2_mma_chunk(const S2Params& p, const S2Smem& sm, int nmt, int warp, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
    const int ng = p.nwp / 8;
    const int pairs = nmt * ng;
    const int p_lo = (warp * pairs) / kWarps, p_hi = ((warp + 1) * pairs) / kWarps;
    int pp = p_lo;
    while (pp < p_hi) {
        const int mtl = pp / ng;
        const int g_lo = pp - mtl * ng;
        const int g_hi = min(ng, g_lo + (p_hi - pp));
        pp += g_hi - g_lo;
        int acc[8][NT][4];
#pragma unroll
        for (int s_ = 0; s_ < 8; ++s_)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[s_][nt][e] = 0;
        const uint32_t* u0 = sm.ublk + (mtl * 16 + gid) * p.su;
        const uint32_t* u1 = u0 + 8 * p.su;
        uint32_t w00 = u0[8 * g_lo + tig], w01 = u0[8 * g_lo + 4 + tig];
        uint32_t w10 = u1[8 * g_lo + tig], w11 = u1[8 * g_lo + 4 + tig];
        for (int g = g_lo; g < g_hi; ++g) {
            const int wb = 8 * g;
            // next group's words, loaded while this group's MMAs issue
            const int wn = (g + 1 < g_hi) ? wb + 8 : wb;
            const uint32_t n00 = u0[wn + tig], n01 = u0[wn + 4 + tig];
            const uint32_t n10 = u1[wn + tig], n11 = u1[wn + 4 + tig];
#pragma unroll
            for (int s_ = 0; s_ < 8; ++s_) {
                const uint32_t msk = 0x01010101u << s_;
                const uint32_t a0 = w00 & msk, a1 = w10 & msk, a2 = w01 & msk, a3 = w11 & msk;
                const uint2* b = reinterpret_cast<const uint2*>(sm.bt) + ((s_ * ng + g) * NT) * 32 + lane;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint2 bb = b[nt * 32];
                    mma_u8s8(acc[s_][nt], a0, a1, a2, a3, bb.x, bb.y);
                }
            }
            w00 = n00; w01 = n01; w10 = n10; w11 = n11;
        }
        // D[row][col]: e = 0,1 -> row gid, cols 2tig, 2tig+1; e = 2,3 -> row gid+8
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                int v = 0;
#pragma unroll
                for (int s_ = 0; s_ < 8; ++s_) v += acc[s_][nt][e] >> s_;
                const int row = mtl * 16 + gid + ((e >> 1) << 3);
                const int col = nt * 8 + 2 * tig + (e & 1);
                atomicAdd(&sm.red[row * (NT * 8) + col], v);
            }
    }
}

// (U t_m) for staged row `row` as 2^-shift (2 P - Tsum), P = d0 + 2^8 d1 + 2^16 d2: exact
// integers times a power of two
template <int NT>
__device__ __forceinline__ double s2_value(const S2Smem& sm, int row, int m, long long tsum, double dinv) {
    const int* rr = sm.red + row * (NT * 8) + 3 * m;
    const long long P = static_cast<long long>(rr[0]) + (static_cast<long long>(rr[1]) << 8) +
                        (static_cast<long long>(rr[2]) << 16);
    return static_cast<double>(2 * P - tsum) * dinv;
}

template <int NT, int TH, int GN, bool PAIR>
__global__ void __launch_bounds__(TH, 1) decode_stage2_kernel(const __grid_constant__ S2Group grp) {
    constexpr int kS2Threads = TH;
    constexpr int kS2Warps = kS2Threads / 32;
    constexpr int NM = PAIR ? 2 : 1;  // members this block works for
    extern __shared__ __align__(16) uint32_t smem2[];
    int li = 0;  // the (first) member of the group this block works for
    if (GN > 1 && !PAIR)
        while (li + 1 < grp.n && static_cast<int>(blockIdx.x) >= grp.cta_off[li + 1]) ++li;
    const int bid = blockIdx.x - grp.cta_off[li];
    const int G = grp.cta_off[li + 1] - grp.cta_off[li];
    S2Smem sm[NM];
    {
        uint32_t* base = smem2;
#pragma unroll
        for (int k = 0; k < NM; ++k) {
            sm[k] = s2_carve<NT>(grp.p[li + k], base);
            base += s2_smem_words<NT>(grp.p[li + k]);
        }
    }
    const S2Params& p = grp.p[li];  // rows, chunking and output of the block (member 0 of a pair)
    __shared__ double s_dinv[NM][NQ_MATVEC_MAX_M];  // 2^-shift: turns the exact integers into values
    __shared__ unsigned long long s_tsum[NM][NQ_MATVEC_MAX_M];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < NM * NQ_MATVEC_MAX_M) s_tsum[tid / NQ_MATVEC_MAX_M][tid % NQ_MATVEC_MAX_M] = 0ull;
    __syncthreads();

    const int mt0 = static_cast<int>((static_cast<int64_t>(bid) * p.mt_total) / G);
    const int mt1 = static_cast<int>((static_cast<int64_t>(bid + 1) * p.mt_total) / G);

    // stage the rows of U of M-tiles [a, b) into ublk (row stride su), for each member; weights
    // only, so this may run before the previous grid has finished
    auto load_u = [&](int a, int b) {
#pragma unroll
        for (int k = 0; k < NM; ++k) {
            const S2Params& q = grp.p[li + k];
            const int64_t row0 = static_cast<int64_t>(a) * 16;
            const int64_t row1 = min(static_cast<int64_t>(b) * 16, q.d_out);
            const int rows = static_cast<int>(row1 - row0);
            // one warp per row, lanes along the row: 16-byte pieces when the row stride allows
            // (reading up to 4 ceil(nw / 4) <= ldu words), else 8- or 4-byte pieces
            const int mode = ((q.ldu & 3) == 0) ? 16 : (((q.ldu & 1) == 0 && (q.nw & 1) == 0) ? 8 : 4);
            const int pieces = mode == 16 ? (q.nw + 3) >> 2 : (mode == 8 ? q.nw >> 1 : q.nw);
            const uint32_t dst0 = static_cast<uint32_t>(__cvta_generic_to_shared(sm[k].ublk));
            const uint32_t* src0 = q.U + row0 * q.ldu;
            for (int rr = warp; rr < rows; rr += kS2Warps) {
                const uint32_t* src = src0 + rr * q.ldu;
                const uint32_t dst = dst0 + 4u * static_cast<uint32_t>(rr * q.su);
                if (mode == 16) {
                    for (int c = lane; c < pieces; c += 32) cp_async16(dst + 16u * c, src + 4 * c);
                } else if (mode == 8) {
                    for (int c = lane; c < pieces; c += 32) cp_async8(dst + 8u * c, src + 2 * c);
                } else {
                    for (int c = lane; c < pieces; c += 32) cp_async4(dst + 4u * c, src + c);
                }
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    // s1 of the same rows (a weight), as fp32, for the epilogue
    auto load_s1 = [&](int a, int b) {
#pragma unroll
        for (int k = 0; k < NM; ++k) {
            const S2Params& q = grp.p[li + k];
            const int64_t row0 = static_cast<int64_t>(a) * 16;
            const int rows = static_cast<int>(min(static_cast<int64_t>(b) * 16, q.d_out) - row0);
            for (int i = tid; i < rows; i += kS2Threads) sm[k].s1_s[i] = f16_bits_to_float(__ldg(q.s1 + row0 + i));
        }
    };

    if (mt0 < mt1) {
        load_u(mt0, min(mt1, mt0 + p.chunk_mt));
        load_s1(mt0, min(mt1, mt0 + p.chunk_mt));
    }
    pdl_launch_dependents();
    pdl_wait();  // t comes from stage 1 of this call

    // ---- t as stage 1 left it: the digit table goes to shared memory as it is (the chunk
    // loop's wait and barrier publish it), the shift and the sum of t_q come from the owners
#pragma unroll
    for (int k = 0; k < NM; ++k) {
        const S2Params& q = grp.p[li + k];
        const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(sm[k].bt));
        const int pieces = 2 * q.nwp * NT * 8;  // 16-byte pieces of 8 nwp NT 8 words
        for (int c = tid; c < pieces; c += kS2Threads) cp_async16(dst + 16u * c, q.tab + 4 * c);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    // warp (k, m) adds member k's row-m owner sums (exact integers), lane 0 keeps the result;
    // each lane issues its loads four at a time, so the sums cost one round trip to L2
    for (int km = warp; km < NM * p.M; km += kS2Warps) {
        const int k = km / p.M, m = km - k * p.M;
        const S2Params& q = grp.p[li + k];
        const int sh = q.tsh[m];
        long long v = 0;
        for (int i0 = lane; i0 < q.tsum_n; i0 += 4 * 32) {
            long long a[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + 32 * u;
                a[u] = (i < q.tsum_n) ? q.tsum[static_cast<int64_t>(i) * q.M + m] : 0ll;
            }
            v += (a[0] + a[1]) + (a[2] + a[3]);
        }
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) {
            s_tsum[k][m] = static_cast<unsigned long long>(v);
            s_dinv[k][m] = pow2_d(-sh);
        }
    }

    for (int c0 = mt0; c0 < mt1; c0 += p.chunk_mt) {
        const int c1 = min(mt1, c0 + p.chunk_mt);
        const int nmt = c1 - c0;
#pragma unroll
        for (int k = 0; k < NM; ++k)
            for (int e = tid; e < nmt * 16 * NT * 8; e += kS2Threads) sm[k].red[e] = 0;
        cp_async_wait_all();
        __syncthreads();
#pragma unroll
        for (int k = 0; k < NM; ++k) s2_mma_chunk<NT, kS2Warps>(grp.p[li + k], sm[k], nmt, warp, lane);
        __syncthreads();

        if (PAIR) {
            // h = silu(g) u from the bf16 gate and up outputs of the same row
            for (int e = tid; e < nmt * 16 * p.M; e += kS2Threads) {
                const int row = (p.M == 1) ? e : e / p.M, m = e - row * p.M;
                const int64_t i = static_cast<int64_t>(c0) * 16 + row;
                if (i < p.d_out) {
                    const double gv = static_cast<double>(sm[0].s1_s[row]) *
                                      s2_value<NT>(sm[0], row, m, static_cast<long long>(s_tsum[0][m]), s_dinv[0][m]);
                    const double uv = static_cast<double>(sm[NM - 1].s1_s[row]) *
                                      s2_value<NT>(sm[NM - 1], row, m, static_cast<long long>(s_tsum[NM - 1][m]),
                                                   s_dinv[NM - 1][m]);
                    p.y[static_cast<int64_t>(m) * p.d_out + i] =
                        silu_mul_bf16(__bfloat16_as_ushort(__double2bfloat16(gv)), __bfloat16_as_ushort(__double2bfloat16(uv)));
                }
            }
        } else if (p.grad) {
            // (U t_m)_i weighted by the cotangent and summed over m in order, in fp64
            for (int row = tid; row < nmt * 16; row += kS2Threads) {
                const int64_t i = static_cast<int64_t>(c0) * 16 + row;
                if (i < p.d_out) {
                    double g = 0.0;
                    for (int m = 0; m < p.M; ++m)
                        g += static_cast<double>(bf16_bits_to_float(p.cot[static_cast<int64_t>(m) * p.d_out + i])) *
                             s2_value<NT>(sm[0], row, m, static_cast<long long>(s_tsum[0][m]), s_dinv[0][m]);
                    p.grad[i] = static_cast<float>(g);
                }
            }
        } else {
            // y = s1 * 2^-shift * (2 P - Tsum)
            for (int e = tid; e < nmt * 16 * p.M; e += kS2Threads) {
                const int row = (p.M == 1) ? e : e / p.M, m = e - row * p.M;
                const int64_t i = static_cast<int64_t>(c0) * 16 + row;
                if (i < p.d_out) {
                    const double yv = static_cast<double>(sm[0].s1_s[row]) *
                                      s2_value<NT>(sm[0], row, m, static_cast<long long>(s_tsum[0][m]), s_dinv[0][m]);
                    p.y[static_cast<int64_t>(m) * p.d_out + i] = __bfloat16_as_ushort(__double2bfloat16(yv));
                }
            }
        }
        __syncthreads();
        if (c1 < mt1) {
            load_u(c1, min(mt1, c1 + p.chunk_mt));
            load_s1(c1, min(mt1, c1 + p.chunk_mt));
        }
    }
    cp_async_wait_all();
}

}  // namespace nq

// ------------------------------------------------------------------------------ host side
#include <atomic>

namespace {

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
constexpr size_t kWsHeader = NQ_WS_HEADER_BYTES;
constexpr size_t kStage1SmemBudget = 200 * 1024;
constexpr size_t kStage2SmemBudget = 200 * 1024;

int ntiles_for(int64_t M) { return static_cast<int>((3 * M + 7) / 8); }

int stage1_max_clusters(int cs);

struct S1Plan {
    int n_chunks, CS, rows_per_slice, jc_rows, zstage;
    size_t smem;
};

int chunks_of(int64_t r) { return static_cast<int>((r / 32 + nq::kS1Words - 1) / nq::kS1Words); }

// Stage-1 shape for a grid of `total_chunks` word chunks over d_in rows: the cluster size CS
// (row slices per chunk, up to 16) is a power of two that keeps the grid near one block per SM,
// raised to any larger size for which the whole grid fits the SMs in one wave with every cluster
// resident at once (the hardware's count of co-resident clusters of that size, one block per
// SM); rows per slice and the staging pass follow.
// A given cluster size (force_cs > 0) replaces the choice, for members of one grid.
S1Plan plan_stage1(int64_t d_in, int total_chunks, int64_t M, int force_cs = 0) {
    S1Plan p{};
    p.n_chunks = total_chunks;
    // more than 8 output columns (M > 2): blocks too register-heavy to share an SM with the
    // previous grid's, so a cluster waits for that many free SMs of one GPC; 8 keeps the wait
    // short (7B attention, M = 8: 30.8 -> 19.1 us per layer against 16)
    const int cap = ntiles_for(M) >= 2 ? 8 : 16;
    // the power of two that keeps the grid near one block per SM, and then any larger size for
    // which the grid still fits the SMs in one wave with every cluster resident at once
    int cs = total_chunks <= 8 ? 16 : (total_chunks <= 18 ? 8 : (total_chunks <= 37 ? 4 : 2));
    while (cs > 1 && static_cast<int64_t>(cs) * 32 > d_in) cs >>= 1;
    if (cs > cap) cs = cap;
    for (int c = cap; c > cs; --c) {
        if (static_cast<int64_t>(c) * 32 > d_in) continue;                               // slices of >= 32 rows
        if (static_cast<int64_t>(c) * total_chunks > nq_host::sm_count()) continue;  // one wave
        if (stage1_max_clusters(c) < total_chunks) continue;  // all clusters resident at once
        cs = c;
        break;
    }
    if (force_cs > 0) cs = force_cs;
    p.CS = cs;
    p.rows_per_slice = static_cast<int>(((d_in + cs - 1) / cs + 31) / 32 * 32);
    const int nt = ntiles_for(M);
    const int swz = nt == 1 ? 8 : 24;
    const size_t fixed = static_cast<size_t>(nq::kS1Outs) * nt * 8 * 4 + static_cast<size_t>(M) * (nq::kS1PartCap + 16) * 8 +
                         nq::kS1Words * 16;
    int64_t jc = static_cast<int64_t>((kStage1SmemBudget - fixed) / (32 + swz)) / 32 * 32;
    if (jc > p.rows_per_slice) jc = p.rows_per_slice;
    if (jc < 32) jc = 32;
    p.jc_rows = static_cast<int>(jc);
    p.smem = static_cast<size_t>(jc) * (32 + swz) + fixed + nq::kS1Words * 16;
    const size_t z_bytes = static_cast<size_t>(M) * (p.rows_per_slice + p.rows_per_slice / 32) * sizeof(float);
    p.zstage = (p.smem + z_bytes <= kStage1SmemBudget && z_bytes <= 48 * 1024) ? 1 : 0;
    if (p.zstage) p.smem += z_bytes;
    return p;
}

// One layer's share of the workspace: stage 2's digit table of t, the owner blocks' sums of
// t_q (room for the largest cluster, 16) and the shifts.
struct TLayout {
    size_t tab, tsum, tsh, total;
};
TLayout t_layout(int64_t r, int64_t M) {
    TLayout o{};
    const int64_t nwp = (r / 32 + 7) / 8 * 8;
    const int nt = ntiles_for(M);
    o.tab = 0;
    o.tsum = align256(static_cast<size_t>(8 * nwp * nt * 8) * 4);
    o.tsh = o.tsum + align256(static_cast<size_t>(chunks_of(r)) * 16 * M * 8);
    o.total = o.tsh + align256(static_cast<size_t>(M) * 4);
    return o;
}

size_t decode_ws_bytes(int64_t r, int64_t M) { return kWsHeader + t_layout(r, M).total; }

// Stage 1 prefetches its rows of V into L2 (off with NQ_DECODE_PREFETCH=0).
bool prefetch_v() {
    static const bool on = [] {
        const char* e = std::getenv("NQ_DECODE_PREFETCH");
        return !(e && e[0] == '0');
    }();
    return on;
}

template <int NT, int TH, int GN>
void set_stage1_attrs_once() {
    static std::atomic<bool> done[64];  // per device; setting an attribute twice is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || done[dev].load(std::memory_order_acquire)) return;
    cudaFuncSetAttribute(nq::decode_stage1_kernel<NT, TH, GN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(kStage1SmemBudget));
    cudaFuncSetAttribute(nq::decode_stage1_kernel<NT, TH, GN>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    done[dev].store(true, std::memory_order_release);
}

template <int NT, int TH, int GN, bool PAIR>
void set_stage2_attrs_once() {
    static std::atomic<bool> done[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || done[dev].load(std::memory_order_acquire)) return;
    cudaFuncSetAttribute(nq::decode_stage2_kernel<NT, TH, GN, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(kStage2SmemBudget));
    done[dev].store(true, std::memory_order_release);
}

// Clusters of cs stage-1 blocks (each holding an SM's shared-memory budget) that can be
// resident at once on this device, from the occupancy query; cached per device and size.
int stage1_max_clusters(int cs) {
    static std::atomic<int> cache[64][17];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || cs < 1 || cs > 16) return 0;
    int v = cache[dev][cs].load(std::memory_order_acquire);
    if (v > 0) return v - 1;
    set_stage1_attrs_once<1, 256, 1>();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, cs);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = kStage1SmemBudget;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = static_cast<unsigned>(cs);
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(nq::decode_stage1_kernel<1, 256, 1>), &cfg) !=
        cudaSuccess) {
        cudaGetLastError();  // leave no error behind; the query is retried on the next call
        return 0;
    }
    cache[dev][cs].store(n + 1, std::memory_order_release);
    return n;
}

// One launch of each stage for n projections that share x (n = 1: a single layer).  With
// `pair` (n = 2, gate and up of equal d_out) stage 2 writes h = silu(gate x) * (up x) to ys[0].
template <int NT, int GN>
nq_status launch_decode_group_nt(const nq_lrb_layer* const* Ls, int n, const uint16_t* x, uint16_t* const* ys, int M,
                                 void* ws, const uint16_t* cot, float* grad, cudaStream_t stream, bool pdl,
                                 float* t_only = nullptr, bool pair = false) {
    // member l's share of the workspace (t's digit table, owner sums, shifts) follows the
    // earlier members'; with t_only (one layer), stage 1 alone runs and writes t in fp32 there
    char* base[nq::kMaxGroup];
    TLayout tl[nq::kMaxGroup];
    size_t off = kWsHeader;
    for (int l = 0; l < n; ++l) {
        tl[l] = t_layout(Ls[l]->r, M);
        base[l] = ws ? static_cast<char*>(ws) + off : nullptr;
        off += tl[l].total;
    }
    int cs1 = 1;  // stage 1's cluster size: owner blocks per word chunk
    {
        int total = 0;
        for (int l = 0; l < n; ++l) total += chunks_of(Ls[l]->r);
        const S1Plan sp = plan_stage1(Ls[0]->d_in, total, M);
        cs1 = sp.CS;
        nq::S1Group g{};
        g.n = n;
        int acc = 0;
        for (int l = 0; l < n; ++l) {
            const nq_lrb_layer* L = Ls[l];
            nq::S1Params& q = g.p[l];
            q.V = L->V;
            q.ldv = L->ldv;
            q.s2 = L->s2;
            q.x = x;
            q.t = t_only;
            if (!t_only) {
                q.tab = reinterpret_cast<uint32_t*>(base[l] + tl[l].tab);
                q.tsum = reinterpret_cast<long long*>(base[l] + tl[l].tsum);
                q.tsh = reinterpret_cast<int*>(base[l] + tl[l].tsh);
            }
            q.nwp = static_cast<int>((L->r / 32 + 7) / 8 * 8);
            q.prefetch = prefetch_v() ? 1 : 0;
            q.M = M;
            q.d_in = L->d_in;
            q.r = static_cast<int>(L->r);
            q.nw = static_cast<int>(L->r / 32);
            q.rows_per_slice = sp.rows_per_slice;
            q.jc_rows = sp.jc_rows;
            q.zstage = sp.zstage;
            g.chunk_off[l] = acc;
            acc += chunks_of(L->r);
        }
        g.chunk_off[n] = acc;
        void* args[] = {&g};
        const bool wide = (NT <= 2) && sp.rows_per_slice >= 1024;
        const void* fn = wide ? reinterpret_cast<const void*>(nq::decode_stage1_kernel<NT, (NT <= 2 ? 512 : 256), GN>)
                              : reinterpret_cast<const void*>(nq::decode_stage1_kernel<NT, 256, GN>);
        if (wide) set_stage1_attrs_once<NT, (NT <= 2 ? 512 : 256), GN>();
        else set_stage1_attrs_once<NT, 256, GN>();
        if (nq_host::launch_ex(fn, dim3(acc, sp.CS), dim3(wide ? 512 : 256), sp.smem, stream, args, pdl, sp.CS) !=
            cudaSuccess)
            return NQ_ERR_LAUNCH;
    }
    if (t_only) return NQ_OK;
    {
        // the SMs are shared among the members in proportion to their weight words; a pair's
        // blocks all work for both members
        const int sms = nq_host::sm_count();
        double wsum = 0.0;
        int mt[nq::kMaxGroup], nwp[nq::kMaxGroup];
        for (int l = 0; l < n; ++l) {
            mt[l] = static_cast<int>((Ls[l]->d_out + 15) / 16);
            nwp[l] = static_cast<int>((Ls[l]->r / 32 + 7) / 8 * 8);
            wsum += static_cast<double>(mt[l]) * nwp[l];
        }
        nq::S2Group g{};
        g.n = n;
        int acc = 0;
        for (int l = 0; l < n; ++l) {
            const nq_lrb_layer* L = Ls[l];
            int gl = pair ? sms : static_cast<int>(sms * (static_cast<double>(mt[l]) * nwp[l]) / wsum + 0.5);
            gl = std::max(1, std::min(gl, mt[l]));
            nq::S2Params& q = g.p[l];
            q.U = L->U;
            q.ldu = L->ldu;
            q.s1 = L->s1;
            q.tab = reinterpret_cast<const uint32_t*>(base[l] + tl[l].tab);
            q.tsum = reinterpret_cast<const long long*>(base[l] + tl[l].tsum);
            q.tsum_n = chunks_of(L->r) * cs1;
            q.tsh = reinterpret_cast<const int*>(base[l] + tl[l].tsh);
            q.y = ys ? ys[l] : nullptr;
            q.cot = cot;
            q.grad = grad;
            q.M = M;
            q.d_out = L->d_out;
            q.r = static_cast<int>(L->r);
            q.nw = static_cast<int>(L->r / 32);
            q.nwp = nwp[l];
            q.su = q.nwp + ((4 - q.nwp % 32) + 32) % 32;
            q.mt_total = mt[l];
            g.cta_off[l] = pair ? 0 : acc;
            if (!pair || l == 0) acc += gl;
        }
        g.cta_off[n] = acc;
        if (pair) g.cta_off[1] = acc;
        // M-tiles staged at a time: a block's whole share when it fits the shared memory
        // (for a pair, both members' rows), else as many as fit
        size_t smem = 0;
        int min_per_cta = 1 << 30;
        {
            const int groups = pair ? 1 : n;
            for (int gi = 0; gi < groups; ++gi) {
                const int l0 = gi, l1 = pair ? n - 1 : gi;
                const int G = g.cta_off[l0 + 1] - g.cta_off[l0];
                const int per_cta = (mt[l0] + G - 1) / G;
                min_per_cta = std::min(min_per_cta, per_cta);
                size_t fixed = 0, per_mt = 0;
                for (int l = l0; l <= l1; ++l) {
                    const nq::S2Params& q = g.p[l];
                    fixed += static_cast<size_t>(8) * q.nwp * NT * 8 * 4;
                    per_mt += static_cast<size_t>(16) * q.su * 4 + static_cast<size_t>(16) * NT * 8 * 4 + 16 * 4;
                }
                int chunk = per_cta;
                if (fixed + chunk * per_mt > kStage2SmemBudget)
                    chunk = static_cast<int>((kStage2SmemBudget - std::min(fixed, kStage2SmemBudget)) / per_mt);
                if (chunk < 1) return NQ_ERR_SHAPE;
                for (int l = l0; l <= l1; ++l) g.p[l].chunk_mt = chunk;
                smem = std::max(smem, fixed + chunk * per_mt);
            }
        }
        void* args[] = {&g};
        const bool wide = (NT == 1) && min_per_cta >= 6;
        const void* fn = nullptr;
        if constexpr (GN > 1) {
            if (pair) {
                fn = wide ? reinterpret_cast<const void*>(nq::decode_stage2_kernel<NT, (NT == 1 ? 512 : 256), GN, true>)
                          : reinterpret_cast<const void*>(nq::decode_stage2_kernel<NT, 256, GN, true>);
                if (wide) set_stage2_attrs_once<NT, (NT == 1 ? 512 : 256), GN, true>();
                else set_stage2_attrs_once<NT, 256, GN, true>();
            }
        }
        if (!fn) {
            fn = wide ? reinterpret_cast<const void*>(nq::decode_stage2_kernel<NT, (NT == 1 ? 512 : 256), GN, false>)
                      : reinterpret_cast<const void*>(nq::decode_stage2_kernel<NT, 256, GN, false>);
            if (wide) set_stage2_attrs_once<NT, (NT == 1 ? 512 : 256), GN, false>();
            else set_stage2_attrs_once<NT, 256, GN, false>();
        }
        if (nq_host::launch_ex(fn, dim3(acc), dim3(wide ? 512 : 256), smem, stream, args, pdl, 1) != cudaSuccess)
            return NQ_ERR_LAUNCH;
    }
    return NQ_OK;
}

// Stage 1 alone for two layers with their own inputs and d_in (a layer and its exchanged form,
// say), as one grid: t0 = V0^T (s2_0 . x0), t1 = V1^T (s2_1 . x1).  The members share the
// cluster size (the smaller of their own choices); each keeps its own row slices.
template <int NT>
nq_status launch_stage1_pair_nt(const nq_lrb_layer* L0, const uint16_t* x0, float* t0, const nq_lrb_layer* L1,
                                const uint16_t* x1, float* t1, int M, cudaStream_t stream, bool pdl) {
    const nq_lrb_layer* Ls[2] = {L0, L1};
    const uint16_t* xs[2] = {x0, x1};
    float* ts[2] = {t0, t1};
    const int total = chunks_of(L0->r) + chunks_of(L1->r);
    const int cs = std::min(plan_stage1(L0->d_in, total, M).CS, plan_stage1(L1->d_in, total, M).CS);
    S1Plan sp[2] = {plan_stage1(L0->d_in, total, M, cs), plan_stage1(L1->d_in, total, M, cs)};
    nq::S1Group g{};
    g.n = 2;
    int acc = 0;
    for (int l = 0; l < 2; ++l) {
        const nq_lrb_layer* L = Ls[l];
        nq::S1Params& q = g.p[l];
        q.V = L->V;
        q.ldv = L->ldv;
        q.s2 = L->s2;
        q.x = xs[l];
        q.t = ts[l];
        q.M = M;
        q.d_in = L->d_in;
        q.r = static_cast<int>(L->r);
        q.nw = static_cast<int>(L->r / 32);
        q.rows_per_slice = sp[l].rows_per_slice;
        q.jc_rows = sp[l].jc_rows;
        q.zstage = sp[l].zstage;
        g.chunk_off[l] = acc;
        acc += chunks_of(L->r);
    }
    g.chunk_off[2] = acc;
    void* args[] = {&g};
    const size_t smem = std::max(sp[0].smem, sp[1].smem);
    const bool wide = (NT <= 2) && std::max(sp[0].rows_per_slice, sp[1].rows_per_slice) >= 1024;
    const void* fn = wide ? reinterpret_cast<const void*>(nq::decode_stage1_kernel<NT, (NT <= 2 ? 512 : 256), nq::kMaxGroup>)
                          : reinterpret_cast<const void*>(nq::decode_stage1_kernel<NT, 256, nq::kMaxGroup>);
    if (wide) set_stage1_attrs_once<NT, (NT <= 2 ? 512 : 256), nq::kMaxGroup>();
    else set_stage1_attrs_once<NT, 256, nq::kMaxGroup>();
    return nq_host::launch_ex(fn, dim3(acc, cs), dim3(wide ? 512 : 256), smem, stream, args, pdl, cs) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_LAUNCH;
}

}  // namespace

size_t nq_decode_workspace_bytes(int64_t d_in, int64_t r, int64_t M) {
    (void)d_in;
    return decode_ws_bytes(r, M);
}

// Shared memory stage 2 needs at the least (its B table plus one staged M-tile of U); the
// caller rejects layers for which this exceeds the budget.
size_t nq_decode_stage2_smem(int64_t r, int64_t M) {
    const int64_t nt = ntiles_for(M);
    const int64_t nwp = (r / 32 + 7) / 8 * 8;
    const int64_t sw = nt * 8;  // B-table columns
    const int64_t su = nwp + ((4 - nwp % 32) + 32) % 32;
    const size_t need = static_cast<size_t>(8 * nwp * sw * 4 + 16 * su * 4 + 16 * nt * 8 * 4 + 16 * 4);
    return need <= kStage2SmemBudget ? need : kStage2SmemBudget + 1;
}

nq_status nq_launch_decode_group(const nq_lrb_layer* const* Ls, int n, const uint16_t* x, uint16_t* const* ys,
                                 int64_t M, void* ws, cudaStream_t stream, bool pdl, const uint16_t* cot,
                                 float* grad) {
    const int m = static_cast<int>(M);
    if (n == 1) {
        switch (ntiles_for(M)) {
            case 1: return launch_decode_group_nt<1, 1>(Ls, n, x, ys, m, ws, cot, grad, stream, pdl);
            case 2: return launch_decode_group_nt<2, 1>(Ls, n, x, ys, m, ws, cot, grad, stream, pdl);
            default: return launch_decode_group_nt<3, 1>(Ls, n, x, ys, m, ws, cot, grad, stream, pdl);
        }
    }
    switch (ntiles_for(M)) {
        case 1: return launch_decode_group_nt<1, nq::kMaxGroup>(Ls, n, x, ys, m, ws, cot, grad, stream, pdl);
        case 2: return launch_decode_group_nt<2, nq::kMaxGroup>(Ls, n, x, ys, m, ws, cot, grad, stream, pdl);
        default: return launch_decode_group_nt<3, nq::kMaxGroup>(Ls, n, x, ys, m, ws, cot, grad, stream, pdl);
    }
}

nq_status nq_launch_decode_gate_up(const nq_lrb_layer* gate, const nq_lrb_layer* up, const uint16_t* x, uint16_t* h,
                                   int64_t M, void* ws, cudaStream_t stream, bool pdl) {
    const nq_lrb_layer* Ls[2] = {gate, up};
    uint16_t* ys[2] = {h, nullptr};
    const int m = static_cast<int>(M);
    switch (ntiles_for(M)) {
        case 1: return launch_decode_group_nt<1, nq::kMaxGroup>(Ls, 2, x, ys, m, ws, nullptr, nullptr, stream, pdl, nullptr, true);
        case 2: return launch_decode_group_nt<2, nq::kMaxGroup>(Ls, 2, x, ys, m, ws, nullptr, nullptr, stream, pdl, nullptr, true);
        default: return launch_decode_group_nt<3, nq::kMaxGroup>(Ls, 2, x, ys, m, ws, nullptr, nullptr, stream, pdl, nullptr, true);
    }
}

// Shared memory the paired stage 2 needs at the least: both digit tables and one M-tile of each.
size_t nq_decode_pair_smem(int64_t r0, int64_t r1, int64_t M) {
    const size_t a = nq_decode_stage2_smem(r0, M), b = nq_decode_stage2_smem(r1, M);
    return (a > kStage2SmemBudget || b > kStage2SmemBudget || a + b > kStage2SmemBudget) ? kStage2SmemBudget + 1 : a + b;
}

nq_status nq_launch_decode(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                           cudaStream_t stream, bool pdl, const uint16_t* cot, float* grad) {
    return nq_launch_decode_group(&L, 1, x, &y, M, ws, stream, pdl, cot, grad);
}

nq_status nq_launch_decode_stage1(const nq_lrb_layer* L, const uint16_t* x, int64_t M, float* t, cudaStream_t stream,
                                  bool pdl) {
    const int m = static_cast<int>(M);
    switch (ntiles_for(M)) {
        case 1: return launch_decode_group_nt<1, 1>(&L, 1, x, nullptr, m, nullptr, nullptr, nullptr, stream, pdl, t);
        case 2: return launch_decode_group_nt<2, 1>(&L, 1, x, nullptr, m, nullptr, nullptr, nullptr, stream, pdl, t);
        default: return launch_decode_group_nt<3, 1>(&L, 1, x, nullptr, m, nullptr, nullptr, nullptr, stream, pdl, t);
    }
}

nq_status nq_launch_decode_stage1_pair(const nq_lrb_layer* L0, const uint16_t* x0, float* t0, const nq_lrb_layer* L1,
                                       const uint16_t* x1, float* t1, int64_t M, cudaStream_t stream, bool pdl) {
    const int m = static_cast<int>(M);
    switch (ntiles_for(M)) {
        case 1: return launch_stage1_pair_nt<1>(L0, x0, t0, L1, x1, t1, m, stream, pdl);
        case 2: return launch_stage1_pair_nt<2>(L0, x0, t0, L1, x1, t1, m, stream, pdl);
        default: return launch_stage1_pair_nt<3>(L0, x0, t0, L1, x1, t1, m, stream, pdl);
    }
}

size_t nq_decode_group_workspace_bytes(const nq_lrb_layer* const* Ls, int n, int64_t M) {
    size_t off = kWsHeader;
    for (int l = 0; l < n; ++l) off += t_layout(Ls[l]->r, M).total;
    return off;
}
