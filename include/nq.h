/*
 * nq.h -- C ABI of the B200 (sm_100a) low-rank binary (LRB) matmul library, libnq.so.
 *
 * The operation (page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language
 * Models", research.samsung.com blog, section 2 "Low-Rank Binary Factorization",
 * factorisation equation):
 *
 *     W ~= s1 (.) (U V^T) (.) s2^T,   U in {-1,+1}^{d_out x r},  V in {-1,+1}^{d_in x r}
 *
 * and the library evaluates, without ever forming W,
 *
 *     y[m][i] = s1_i * sum_k U_ik * ( sum_j V_jk * s2_j * x[m][j] )
 *
 * for M rows of activations x.  The sign factors are stored as packed bits (section 3,
 * "Phase 3: Scale-Only Model Reconstruction": frozen binary factors packed into integer
 * formats).
 *
 * Conventions for every entry point
 * ---------------------------------
 * - Tensor pointers are DEVICE pointers on the current CUDA device, owned by the caller.
 *   The library never allocates or frees device memory, never synchronises the stream
 *   (except nq_sync_status) and keeps no state between calls besides one device error word
 *   per device.  Calls on different streams may run concurrently as long as they do not
 *   share a workspace.
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 * - Packed sign layout: row i of a [rows][ld] uint32 matrix holds element k of that row at
 *   bit (k % 32) of word (k / 32), least significant bit first; bit 1 means +1, bit 0
 *   means -1.  r must be a multiple of 32.  Words r/32 .. ld-1 of a row are padding: pack
 *   writes them as 0, and their values never affect a result (the decode kernels may copy
 *   them along with the row).
 * - fp16 values (s1, s2) and bf16 values (x, y) are passed as uint16_t bit patterns.
 * - Activations are row-major: x is [M][d_in], y is [M][d_out], contiguous.
 * - Alignment: every pointer must be 16-byte aligned (NQ_ERR_ALIGN otherwise).
 * - Arguments are validated on the host before anything is launched; on an error nothing
 *   is launched and outputs are untouched.
 * - Kernels read the weights (U, V, s1, s2) before they wait for the work queued ahead of
 *   them on the stream (programmatic dependent launch): the caller must not write a
 *   layer's weights in the kernel launched immediately before a call that reads them
 *   without a stream/event synchronisation in between.  Activations and workspace are
 *   only touched after that wait.
 * - Environment: NQ_DISABLE_PDL=1 launches every kernel without programmatic dependent
 *   launch (each waits for the previous grid in full); NQ_DECODE_PREFETCH=0 stops the decode
 *   stage 1 from asking the copy engine to prefetch its rows of V into L2.  Both are read once
 *   per process and change timing only, never a result.
 */
#ifndef NQ_H_
#define NQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported from libnq.so (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define NQ_API __attribute__((visibility("default")))
#else
#define NQ_API
#endif

typedef enum nq_status {
    NQ_OK = 0,
    NQ_ERR_NULL = 1,      /* a required pointer is NULL */
    NQ_ERR_SHAPE = 2,     /* non-positive size, r % 32 != 0, ld too small, M out of range */
    NQ_ERR_ALIGN = 3,     /* a pointer is not 16-byte aligned */
    NQ_ERR_WORKSPACE = 4, /* workspace NULL or smaller than nq_workspace_bytes() */
    NQ_ERR_DEVICE = 5,    /* current device is not compute capability 10.0 (B200) */
    NQ_ERR_LAUNCH = 6,    /* a kernel launch failed */
    NQ_ERR_TIMEOUT = 7,   /* a bounded device-side wait gave up (seen by nq_sync_status) */
    NQ_ERR_SCRATCH_LIMIT = 8 /* nq_lrb_matvec_noalloc: the call needs more than NQ_NOALLOC_SCRATCH_BYTES */
} nq_status;

/* One LRB linear layer.  All pointers are device pointers; the struct itself is host
 * memory and is read only during the call. */
typedef struct nq_lrb_layer {
    int64_t d_out;      /* output features (rows of U, length of s1) */
    int64_t d_in;       /* input features (rows of V, length of s2) */
    int64_t r;          /* rank, a multiple of 32, at most NQ_MAX_RANK_LIMIT */
    const uint32_t* U;  /* [d_out][ldu] packed signs of U */
    int64_t ldu;        /* words per row of U, >= r/32 */
    const uint32_t* V;  /* [d_in][ldv] packed signs of V */
    int64_t ldv;        /* words per row of V, >= r/32 */
    const uint16_t* s1; /* [d_out] fp16 */
    const uint16_t* s2; /* [d_in] fp16 */
} nq_lrb_layer;

/* Largest rank any entry point accepts. */
#define NQ_MAX_RANK_LIMIT 262144

/* Largest row count nq_lrb_matvec accepts (the decode path). */
#define NQ_MATVEC_MAX_M 8

/*
 * nq_pack_signs -- sign extraction and bit packing of latent factors.
 * Section 3 "Step 3: Factorized Component Refinement" (the binary factors are sign(U),
 * sign(V) of latent matrices) and "Phase 3" (frozen signs packed into integers).
 *   latent    [rows][ld_latent] fp32, device; columns 0..r-1 are read.
 *   packed    [rows][ld_words] uint32, device; written in full (pad words = 0).
 *   bit(i,k) = (latent[i][k] >= 0): +0 and -0 give 1, NaN gives 0, +-inf by sign.
 * Requires rows >= 0, r >= 0, r % 32 == 0, ld_latent >= r, ld_words >= r/32.  rows == 0
 * or r == 0 with ld_words == 0 is a no-op.  Bit-exact and deterministic.
 */
NQ_API nq_status nq_pack_signs(const float* latent, int64_t rows, int64_t r, int64_t ld_latent, uint32_t* packed,
                        int64_t ld_words, void* stream);

/*
 * nq_workspace_bytes -- device scratch a call with M activation rows needs (for
 * nq_lrb_matvec, nq_lrb_matmul, nq_layer_forward, nq_lrb_transposed and
 * nq_lrb_scale_grads alike).  Returns 0 for an invalid layer or M.  The workspace must stay
 * untouched by other work while the call runs.  Its first 4096 bytes are a reserved header
 * that the kernels neither read nor write; the rest is per-call scratch, fully written
 * before it is read.  So one workspace can be reused by consecutive calls of any shape on
 * the same stream, with no initialisation.
 */
NQ_API size_t nq_workspace_bytes(const nq_lrb_layer* L, int64_t M);

/*
 * nq_lrb_matvec -- decode path, 1 <= M <= NQ_MATVEC_MAX_M.
 * Section 2 factorisation equation, evaluated as two streaming stages over the packed
 * words: t[m][k] = sum_j V_jk s2_j x[m][j], then y[m][i] = bf16(s1_i sum_k U_ik t[m][k]).
 *   x [M][d_in] bf16, y [M][d_out] bf16 (round to nearest even), ws = workspace of at
 *   least nq_workspace_bytes(L, M) bytes (16-byte aligned).
 * Both stages sum exact integers: s2 x is quantised to 23-bit fixed point per row slice of V,
 * t to 23-bit fixed point per batch row (the shift from an exact bound on |t|), and the
 * partial sums are combined in fp64 in a fixed order.  Results are run-to-run deterministic.
 * Finite results need |s2_j x[m][j]| within the fp32 range.
 */
NQ_API nq_status nq_lrb_matvec(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                        size_t ws_bytes, void* stream);

/*
 * nq_lrb_matmul -- prefill path on the tensor cores (tcgen05), any M >= 1 (tuned for
 * M >= 64).  Same operation as nq_lrb_matvec.  The activations are scaled by s2 and by one
 * power of two 2^-e_m per row m, chosen so that sum_j |2^-e_m x_mj s2_j| <= 2^14, and rounded
 * to fp16; the packed signs are expanded to fp16 +-1 on chip; both products accumulate in fp32
 * (TMEM); the intermediate t (|t| <= 2^14 by the choice of e_m) is rounded to fp16; y is scaled
 * back by 2^e_m and s1 and rounded to bf16.  So no finite bf16 input overflows fp16 on the way,
 * rows of very small values keep fp16's full precision, and y is finite whenever its value
 * lies in the bf16 range.  The powers of two are exact: rows that stay inside fp16's normal
 * range either way give the same bits as without them.  The workspace holds e_m.
 */
NQ_API nq_status nq_lrb_matmul(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                        size_t ws_bytes, void* stream);

/* nq_layer_forward -- M <= NQ_MATVEC_MAX_M: nq_lrb_matvec; otherwise nq_lrb_matmul. */
NQ_API nq_status nq_layer_forward(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * nq_lrb_from_latent -- a packed layer from its latent factors.  Page "NanoQuant: Efficient
 * Sub-1-Bit Quantization of Large Language Models", section 3, "Magnitude Balancing and Scale
 * Extraction", then "Phase 3" packing.  For the continuous proxies Uh [d_out][ld_uh] and
 * Vh [d_in][ld_vh] (fp32, r columns each):
 *     eta = sqrt( ||Vh||_F / ||Uh||_F )   (1 when either norm is 0),
 *     U := eta Uh,  V := Vh / eta,  s1_i = mean_k |U_ik|,  s2_j = mean_k |V_jk|,
 * and the binary factors sign(U), sign(V) packed as nq_pack_signs does (eta > 0, so the signs
 * are those of Uh, Vh).  Outputs (device, caller-owned): U [d_out][ldu], V [d_in][ldv] words,
 * s1 [d_out], s2 [d_in] fp16 bit patterns (round to nearest even), and eta (one double; may be
 * NULL).  Norms and means are summed in fp64 in a fixed order (run-to-run identical).
 * ws: nq_from_latent_workspace_bytes(d_out, d_in, r, ldu, ldv) bytes.
 */
NQ_API size_t nq_from_latent_workspace_bytes(int64_t d_out, int64_t d_in, int64_t r, int64_t ldu, int64_t ldv);
NQ_API nq_status nq_lrb_from_latent(const float* Uh, int64_t ld_uh, const float* Vh, int64_t ld_vh, int64_t d_out,
                                    int64_t d_in, int64_t r, uint32_t* U, int64_t ldu, uint32_t* V, int64_t ldv,
                                    uint16_t* s1, uint16_t* s2, double* eta, void* ws, size_t ws_bytes,
                                    void* stream);

/*
 * Calibration products.  Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language
 * Models", section 3, "Phase 3: Scale-Only Model Reconstruction": with U and V frozen and
 * packed, only s1 and s2 are optimised, so a training step needs the layer's transpose (to
 * carry the output gradient to the layer's input) and the gradients with respect to the two
 * scale vectors.  Both come from the section 2 equation read elementwise,
 * W_ij = s1_i (sum_k U_ik V_jk) s2_j.
 *
 * nq_lrb_transposed -- xbar[m][j] = bf16( sum_i W_ij ybar[m][i] )
 *                                = bf16( s2_j sum_k V_jk sum_i U_ik s1_i ybar[m][i] ).
 *   ybar [M][d_out] bf16 (the cotangent of y), xbar [M][d_in] bf16.  Computed as the forward
 *   product of the layer with (U, s1, d_out) and (V, s2, d_in) exchanged: M <= NQ_MATVEC_MAX_M
 *   on the decode path, larger M on the tensor cores, with the same numerics as
 *   nq_lrb_matvec and nq_lrb_matmul respectively.  ws: nq_workspace_bytes(L, M) bytes.
 */
NQ_API nq_status nq_lrb_transposed(const nq_lrb_layer* L, const uint16_t* ybar, uint16_t* xbar, int64_t M, void* ws,
                                   size_t ws_bytes, void* stream);

/*
 * nq_lrb_scale_grads -- for L = sum_m sum_i ybar[m][i] y[m][i], y = the layer applied to x:
 *   g_s1[i] = dL/ds1_i = sum_m ybar[m][i] sum_k U_ik t[m][k],  t[m] = V^T (s2 . x[m])
 *   g_s2[j] = dL/ds2_j = sum_m x[m][j]    sum_k V_jk u[m][k],  u[m] = U^T (s1 . ybar[m])
 *   x [M][d_in] and ybar [M][d_out] bf16; g_s1 [d_out] and g_s2 [d_in] fp32, overwritten
 *   (16-byte aligned).  M <= NQ_MATVEC_MAX_M: the decode kernels' exact integer sums of the
 *   23-bit quantised activations, weighted by the cotangent and summed over m in fp64.
 *   Larger M: the tensor-core products (fp16 operands, fp32 accumulation), weighted and summed
 *   over tokens in fp64, token tiles in a fixed order: run-to-run identical.
 *   ws: nq_workspace_bytes(L, M) bytes.
 */
NQ_API nq_status nq_lrb_scale_grads(const nq_lrb_layer* L, const uint16_t* x, const uint16_t* ybar, int64_t M,
                                    float* g_s1, float* g_s2, void* ws, size_t ws_bytes, void* stream);

/*
 * Gradients with respect to the sign factors.  Page "NanoQuant: Efficient Sub-1-Bit
 * Quantization of Large Language Models", section 3, "Step 3: Factorized Component
 * Refinement": the latent factors are refined through sign() with straight-through
 * estimators.  For L = sum_m sum_i ybar[m][i] y[m][i] (y = the layer applied to x):
 *   gU[i][k] = dL/dU_ik = s1_i sum_m ybar[m][i] t[m][k],  t[m] = V^T (s2 . x[m])
 *   gV[j][k] = dL/dV_jk = s2_j sum_m x[m][j]    u[m][k],  u[m] = U^T (s1 . ybar[m])
 * The identity straight-through estimator passes these to the latent entries unchanged
 * (the pages name no variant); a clipped estimator is the caller's mask on gU, gV.
 *   x [M][d_in], ybar [M][d_out] bf16; gU [d_out][ldgu] and gV [d_in][ldgv] fp32, columns
 *   0..r-1 overwritten, pad columns untouched.  ldgu, ldgv >= r and multiples of 4; gU, gV
 *   16-byte aligned (NQ_ERR_ALIGN otherwise).
 *   M <= NQ_MATVEC_MAX_M: t and u from the decode stage 1 (exact integer sums of the 23-bit
 *   quantised activations, fp32), the sum over m in fp32 on the CUDA cores.  Larger M: t and u
 *   from the tensor-core GEMM 1 (fp16 operands s2 . x and s1 . ybar, fp16 t, u), the sum over
 *   m on the tensor cores (fp16 operands, fp32 accumulation).  That sum runs over the rows,
 *   so they share one scale: finite results here need |x_j s2_j|, |ybar_i s1_i|, |t_k| and
 *   |u_k| below the fp16 range (65504).
 *   ws: nq_sign_grads_workspace_bytes(L, M) bytes (0 for an invalid layer or M < 1).
 */
NQ_API size_t nq_sign_grads_workspace_bytes(const nq_lrb_layer* L, int64_t M);
NQ_API nq_status nq_lrb_sign_grads(const nq_lrb_layer* L, const uint16_t* x, const uint16_t* ybar, int64_t M,
                                   float* gU, int64_t ldgu, float* gV, int64_t ldgv, void* ws, size_t ws_bytes,
                                   void* stream);

/*
 * nq_layer_forward_group -- y[l] = layer l applied to x, for 1 <= n <= NQ_MAX_GROUP projections
 * that share their input (a transformer's q, k, v, or its gate and up): every layer must have
 * the same d_in; d_out and r may differ.  For M <= NQ_MATVEC_MAX_M the group runs as one
 * launch of each decode stage (the layers' blocks side by side), which saves a kernel pair's
 * fixed latency per extra member; numerics as nq_lrb_matvec, except that the row slices of V
 * over which x is quantised follow the group's total size.  Larger M runs nq_lrb_matmul once
 * per layer.  y: array of n output pointers ([M][d_out_l] bf16 each); ws:
 * nq_group_workspace_bytes(layers, n, M) bytes (0 for an invalid group).
 */
#define NQ_MAX_GROUP 4
NQ_API size_t nq_group_workspace_bytes(const nq_lrb_layer* const* layers, int n, int64_t M);
NQ_API nq_status nq_layer_forward_group(const nq_lrb_layer* const* layers, int n, const uint16_t* x,
                                        uint16_t* const* y, int64_t M, void* ws, size_t ws_bytes, void* stream);

/*
 * nq_mlp_gate_up -- h = bf16( silu(bf16(gate x)) * bf16(up x) ) for the gate and up projections
 * of a Llama MLP block built from LRB layers (the pages quantise each projection on its own;
 * the block around them is not part of the factorisation).  gate and up share x: equal d_in
 * and equal d_out, r may differ.  The result equals, bit for bit, nq_layer_forward_group on
 * {gate, up} followed by nq_silu_mul of its two outputs, but for M <= NQ_MATVEC_MAX_M the gate
 * and up outputs never reach memory: stage 2 of the grouped decode computes both projections of
 * a row in the same block and applies SiLU.mul in its epilogue, one launch fewer per MLP block.
 * Larger M (or ranks whose two stage-2 tables do not fit on chip together) runs the unfused
 * calls, with the two outputs kept in the workspace.  x [M][d_in], h [M][d_out] bf16, device,
 * 16-byte aligned; ws: nq_mlp_gate_up_workspace_bytes(gate, up, M) bytes (0 for invalid
 * layers or M < 1).  Errors: NQ_ERR_NULL, NQ_ERR_ALIGN, NQ_ERR_SHAPE (d_in or d_out differ,
 * M < 1, a layer too large for the decode path), NQ_ERR_WORKSPACE, NQ_ERR_DEVICE.
 */
NQ_API size_t nq_mlp_gate_up_workspace_bytes(const nq_lrb_layer* gate, const nq_lrb_layer* up, int64_t M);
NQ_API nq_status nq_mlp_gate_up(const nq_lrb_layer* gate, const nq_lrb_layer* up, const uint16_t* x, uint16_t* h,
                                int64_t M, void* ws, size_t ws_bytes, void* stream);

/*
 * nq_silu_mul -- h[e] = bf16( silu(g[e]) * u[e] ), silu(g) = g / (1 + exp(-g)), fp32 math,
 * for the Llama MLP block built from LRB projections (gate, up -> h -> down).  Not part of
 * the factorisation itself.  g, u, h: n bf16 values each, device.
 */
NQ_API nq_status nq_silu_mul(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t n, void* stream);

/*
 * nq_sync_status -- synchronises `stream`, then reports and clears this device's error
 * word: NQ_ERR_TIMEOUT if a bounded device-side wait gave up since the last check,
 * NQ_ERR_LAUNCH if the stream reported an asynchronous CUDA error, NQ_OK otherwise.
 */
NQ_API nq_status nq_sync_status(void* stream);

/*
 * nq_selftest_bounded_wait -- exercises the failure path of the library's bounded device waits
 * (diagnostic; never needed in normal use).  Launches one block on `stream` whose thread waits,
 * for limit_us microseconds (1000 .. 2000000, NQ_ERR_SHAPE otherwise), on an mbarrier that
 * nothing completes.  The wait gives up, records the timeout in the device error word and the
 * kernel exits normally, so the context stays usable; the next nq_sync_status returns
 * NQ_ERR_TIMEOUT and clears the word.  NQ_ERR_DEVICE on a device that is not sm_100.
 */
NQ_API nq_status nq_selftest_bounded_wait(int64_t limit_us, void* stream);

/*
 * nq_lrb_matvec_noalloc -- nq_lrb_matvec for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it exists for deployment.  Callers that
 * cannot hand over a workspace: plug-ins that an inference engine gives only their input and
 * output tensors, latency-critical loops that cannot take an allocator round trip, plain C
 * callers without an allocator.
 * Same operation, arguments, validation and numerics as nq_lrb_matvec, minus the workspace:
 * the scratch (t's digit table and its sums) lives in one statically sized array of
 * NQ_NOALLOC_SCRATCH_BYTES inside libnq.so, which every GPU that loads the library holds until
 * the process exits.  Every shape that the decode kernels accept fits in it: stage 2's shared
 * memory caps r (20224 at M <= 2, 11264 at M <= 5, 7680 at M <= 8), and the scratch such a
 * layer needs stays under 256 KB.  Should a later layout need more than the array holds, the
 * call returns NQ_ERR_SCRATCH_LIMIT without launching.  The decode kernels
 * write all of the scratch they read, so nothing in the array has to start at zero.
 * The first call on a device looks up the array's device address (set-up, with that device
 * current; a failed look-up returns NQ_ERR_LAUNCH and is tried again on the next call); make
 * that first call before any stream capture.
 * All calls on a device share the one array: calls that can overlap on the GPU (different
 * streams, or the same stream without ordering) race and must be serialised by the caller.
 * Never calls cudaMalloc, cudaFree or any allocating routine.
 */
#define NQ_NOALLOC_SCRATCH_BYTES (2u * 1024u * 1024u)
NQ_API nq_status nq_lrb_matvec_noalloc(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M,
                                       void* stream);

/* Human-readable name of a status code (static storage). */
NQ_API const char* nq_status_string(nq_status s);

/* Library build identification (static storage): target architecture and version. */
NQ_API const char* nq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NQ_H_ */
