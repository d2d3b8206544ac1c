// api.cu -- the C ABI declared in include/nq.h: argument validation, device checks,
// workspace planning and dispatch to the kernels.  No allocation, no synchronisation (except
// nq_sync_status), no fallback: a device that is not sm_100 gets NQ_ERR_DEVICE.
#include <algorithm>
#include <mutex>

#include "nq_common.cuh"

namespace nq {
__device__ unsigned int g_error_word = 0u;
}

// kernels' host launchers (defined next to each kernel)
nq_status nq_launch_pack(const float*, int64_t, int64_t, int64_t, uint32_t*, int64_t, cudaStream_t);
size_t nq_decode_workspace_bytes(int64_t d_in, int64_t r, int64_t M);
size_t nq_decode_stage2_smem(int64_t r, int64_t M);
nq_status nq_launch_silu_mul(const uint16_t*, const uint16_t*, uint16_t*, int64_t, cudaStream_t, bool);
size_t nq_prefill_workspace_bytes(const nq_lrb_layer*, int64_t M);
size_t nq_decode_pair_smem(int64_t r0, int64_t r1, int64_t M);
nq_status nq_launch_decode_gate_up(const nq_lrb_layer* gate, const nq_lrb_layer* up, const uint16_t* x, uint16_t* h,
                                   int64_t M, void* ws, cudaStream_t stream, bool pdl);
size_t nq_from_latent_ws(int64_t d_out, int64_t d_in, int64_t ldu, int64_t ldv);
nq_status nq_launch_from_latent(const float* Uh, int64_t ld_uh, const float* Vh, int64_t ld_vh, int64_t d_out,
                                int64_t d_in, int64_t r, uint32_t* U, int64_t ldu, uint32_t* V, int64_t ldv,
                                uint16_t* s1, uint16_t* s2, double* eta, void* ws, cudaStream_t stream);
size_t nq_sign_grads_ws(const nq_lrb_layer* L, const nq_lrb_layer* X, int64_t M);
nq_status nq_launch_sign_grads(const nq_lrb_layer* L, const nq_lrb_layer* X, const uint16_t* x, const uint16_t* ybar,
                               int64_t M, float* gU, int64_t ldgu, float* gV, int64_t ldgv, void* ws,
                               cudaStream_t stream, bool pdl);

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kMaxDecodeSmem = 200 * 1024;

struct DeviceInfo {
    std::once_flag once;
    bool ok = false;
    int sms = 0;
    unsigned int* err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];

// Returns the current device's info, probing it once.  ok == false: not sm_100.
DeviceInfo* current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    DeviceInfo* d = &g_dev[dev];
    std::call_once(d->once, [d, dev]() {
        int major = 0, minor = 0, sms = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        d->sms = sms;
        d->ok = (major == 10 && minor == 0 && sms > 0);
        void* p = nullptr;
        if (d->ok && cudaGetSymbolAddress(&p, nq::g_error_word) == cudaSuccess) d->err = static_cast<unsigned int*>(p);
        d->ok = d->ok && d->err != nullptr;
    });
    return d;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pdl_enabled() {
    static const bool on = [] {
        const char* e = getenv("NQ_DISABLE_PDL");
        return !(e && e[0] == '1');
    }();
    return on;
}

nq_status check_layer(const nq_lrb_layer* L) {
    if (!L || !L->U || !L->V || !L->s1 || !L->s2) return NQ_ERR_NULL;
    if (L->d_out <= 0 || L->d_in <= 0 || L->r <= 0 || (L->r % 32) != 0) return NQ_ERR_SHAPE;
    if (L->ldu < L->r / 32 || L->ldv < L->r / 32 || L->r > NQ_MAX_RANK) return NQ_ERR_SHAPE;
    if (!aligned16(L->U) || !aligned16(L->V) || !aligned16(L->s1) || !aligned16(L->s2)) return NQ_ERR_ALIGN;
    return NQ_OK;
}

nq_status check_io(const uint16_t* x, const uint16_t* y, void* ws) {
    if (!x || !y || !ws) return NQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(y) || !aligned16(ws)) return NQ_ERR_ALIGN;
    return NQ_OK;
}

// The layer with the roles of (U, s1, d_out) and (V, s2, d_in) exchanged: its forward product
// is the transpose of L's, since W_ij = s1_i G_ij s2_j and G_ij = G^T_ji.
nq_lrb_layer exchanged(const nq_lrb_layer* L) {
    nq_lrb_layer T = *L;
    T.d_out = L->d_in;
    T.d_in = L->d_out;
    T.U = L->V;
    T.ldu = L->ldv;
    T.V = L->U;
    T.ldv = L->ldu;
    T.s1 = L->s2;
    T.s2 = L->s1;
    return T;
}

}  // namespace

namespace nq_host {

bool pdl_on() { return pdl_enabled(); }

nq_status check_decode_call(const nq_lrb_layer* L, int64_t M) {
    nq_status st = check_layer(L);
    if (st != NQ_OK) return st;
    if (M < 1 || M > NQ_MATVEC_MAX_M) return NQ_ERR_SHAPE;
    if (nq_decode_stage2_smem(L->r, M) > kMaxDecodeSmem) return NQ_ERR_SHAPE;
    return NQ_OK;
}

bool device_ready() {
    DeviceInfo* d = current_device();
    return d && d->ok;
}

int sm_count() {
    DeviceInfo* d = current_device();
    return (d && d->sms > 0) ? d->sms : 148;
}

unsigned int* error_word() {
    DeviceInfo* d = current_device();
    return d ? d->err : nullptr;
}

cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s, void** args, bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_ex(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s, void** args, bool pdl,
                      int cluster_y) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_y > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = 1;
        attr[n].val.clusterDim.y = static_cast<unsigned>(cluster_y);
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace nq_host

extern "C" {

const char* nq_status_string(nq_status s) {
    switch (s) {
        case NQ_OK: return "NQ_OK";
        case NQ_ERR_NULL: return "NQ_ERR_NULL: a required pointer is NULL";
        case NQ_ERR_SHAPE: return "NQ_ERR_SHAPE: invalid size, rank or leading dimension";
        case NQ_ERR_ALIGN: return "NQ_ERR_ALIGN: a pointer is not 16-byte aligned";
        case NQ_ERR_WORKSPACE: return "NQ_ERR_WORKSPACE: workspace missing or too small";
        case NQ_ERR_DEVICE: return "NQ_ERR_DEVICE: current device is not sm_100 (B200)";
        case NQ_ERR_LAUNCH: return "NQ_ERR_LAUNCH: kernel launch or asynchronous CUDA error";
        case NQ_ERR_TIMEOUT: return "NQ_ERR_TIMEOUT: a bounded device-side wait gave up";
        case NQ_ERR_SCRATCH_LIMIT:
            return "NQ_ERR_SCRATCH_LIMIT: the call needs more scratch than nq_lrb_matvec_noalloc's static array";
    }
    return "unknown nq_status";
}

const char* nq_version(void) { return "libnq 0.1 sm_100a"; }

nq_status nq_pack_signs(const float* latent, int64_t rows, int64_t r, int64_t ld_latent, uint32_t* packed,
                        int64_t ld_words, void* stream) {
    if (rows < 0 || r < 0 || (r % 32) != 0 || ld_latent < r || ld_words < r / 32) return NQ_ERR_SHAPE;
    if (rows == 0 || ld_words == 0) return NQ_OK;
    if (!packed || (r > 0 && !latent)) return NQ_ERR_NULL;
    if (!aligned16(packed) || (latent && !aligned16(latent))) return NQ_ERR_ALIGN;
    DeviceInfo* d = current_device();
    if (!d || !d->ok) return NQ_ERR_DEVICE;
    return nq_launch_pack(latent, rows, r, ld_latent, packed, ld_words, static_cast<cudaStream_t>(stream));
}

size_t nq_workspace_bytes(const nq_lrb_layer* L, int64_t M) {
    if (check_layer(L) != NQ_OK || M < 1) return 0;
    // one workspace serves the forward product, the transpose and the scale gradients
    const nq_lrb_layer T = exchanged(L);
    size_t bytes = nq_prefill_workspace_bytes(L, M);
    const size_t bytes_t = nq_prefill_workspace_bytes(&T, M);
    if (bytes_t > bytes) bytes = bytes_t;
    if (M <= NQ_MATVEC_MAX_M) {
        const size_t dec = nq_decode_workspace_bytes(L->d_in, L->r, M);
        if (dec > bytes) bytes = dec;
    }
    return bytes;
}

nq_status nq_lrb_matvec(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                        size_t ws_bytes, void* stream) {
    nq_status st = nq_host::check_decode_call(L, M);
    if (st != NQ_OK) return st;
    if ((st = check_io(x, y, ws)) != NQ_OK) return st;
    if (ws_bytes < nq_decode_workspace_bytes(L->d_in, L->r, M)) return NQ_ERR_WORKSPACE;
    DeviceInfo* d = current_device();
    if (!d || !d->ok) return NQ_ERR_DEVICE;
    return nq_launch_decode(L, x, y, M, ws, static_cast<cudaStream_t>(stream), pdl_enabled());
}

nq_status nq_lrb_matmul(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                        size_t ws_bytes, void* stream) {
    nq_status st = check_layer(L);
    if (st != NQ_OK) return st;
    if (M < 1) return NQ_ERR_SHAPE;
    if ((st = check_io(x, y, ws)) != NQ_OK) return st;
    if (ws_bytes < nq_prefill_workspace_bytes(L, M)) return NQ_ERR_WORKSPACE;
    DeviceInfo* d = current_device();
    if (!d || !d->ok) return NQ_ERR_DEVICE;
    return nq_launch_prefill(L, x, y, M, ws, static_cast<cudaStream_t>(stream), pdl_enabled());
}

nq_status nq_layer_forward(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M, void* ws,
                           size_t ws_bytes, void* stream) {
    if (M >= 1 && M <= NQ_MATVEC_MAX_M) return nq_lrb_matvec(L, x, y, M, ws, ws_bytes, stream);
    return nq_lrb_matmul(L, x, y, M, ws, ws_bytes, stream);
}

size_t nq_group_workspace_bytes(const nq_lrb_layer* const* layers, int n, int64_t M) {
    if (!layers || n < 1 || n > NQ_MAX_GROUP || M < 1) return 0;
    size_t bytes = 0;
    for (int l = 0; l < n; ++l) {
        if (check_layer(layers[l]) != NQ_OK || layers[l]->d_in != layers[0]->d_in) return 0;
        bytes = std::max(bytes, nq_workspace_bytes(layers[l], M));
    }
    if (M <= NQ_MATVEC_MAX_M) bytes = std::max(bytes, nq_decode_group_workspace_bytes(layers, n, M));
    return bytes;
}

nq_status nq_layer_forward_group(const nq_lrb_layer* const* layers, int n, const uint16_t* x, uint16_t* const* y,
                                 int64_t M, void* ws, size_t ws_bytes, void* stream) {
    if (!layers || !y) return NQ_ERR_NULL;
    if (n < 1 || n > NQ_MAX_GROUP || M < 1) return NQ_ERR_SHAPE;
    nq_status st;
    for (int l = 0; l < n; ++l) {
        if ((st = check_layer(layers[l])) != NQ_OK) return st;
        if (layers[l]->d_in != layers[0]->d_in) return NQ_ERR_SHAPE;
        if (M <= NQ_MATVEC_MAX_M && nq_decode_stage2_smem(layers[l]->r, M) > kMaxDecodeSmem) return NQ_ERR_SHAPE;
        if ((st = check_io(x, y[l], ws)) != NQ_OK) return st;
    }
    if (ws_bytes < nq_group_workspace_bytes(layers, n, M)) return NQ_ERR_WORKSPACE;
    DeviceInfo* d = current_device();
    if (!d || !d->ok) return NQ_ERR_DEVICE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M <= NQ_MATVEC_MAX_M) return nq_launch_decode_group(layers, n, x, y, M, ws, s, pdl_enabled());
    for (int l = 0; l < n; ++l)
        if ((st = nq_launch_prefill(layers[l], x, y[l], M, ws, s, pdl_enabled())) != NQ_OK) return st;
    return NQ_OK;
}

nq_status nq_lrb_transposed(const nq_lrb_layer* L, const uint16_t* ybar, uint16_t* xbar, int64_t M, void* ws,
                            size_t ws_bytes, void* stream) {
    nq_status st = check_layer(L);
    if (st != NQ_OK) return st;
    if (M < 1) return NQ_ERR_SHAPE;
    if (M <= NQ_MATVEC_MAX_M && nq_decode_stage2_smem(L->r, M) > kMaxDecodeSmem) return NQ_ERR_SHAPE;
    if ((st = check_io(ybar, xbar, ws)) != NQ_OK) return st;
    if (ws_bytes < nq_workspace_bytes(L, M)) return NQ_ERR_WORKSPACE;
    DeviceInfo* d = current_device();
    if (!d || !d->ok) return NQ_ERR_DEVICE;
    const nq_lrb_layer T = exchanged(L);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M <= NQ_MATVEC_MAX_M) return nq_launch_decode(&T, ybar, xbar, M, ws, s, pdl_enabled());
    return nq_launch_prefill(&T, ybar, xbar, M, ws, s, pdl_enabled());
}

nq_status nq_lrb_scale_grads(const nq_lrb_layer* L, const uint16_t* x, const uint16_t* ybar, int64_t M, float* g_s1,
                             float* g_s2, void* ws, size_t ws_bytes, void* stream) {
    nq_status st = check_layer(L);
    if (st != NQ_OK) return st;
    if (M < 1) return NQ_ERR_SHAPE;
    if (M <= NQ_MATVEC_MAX_M && nq_decode_stage2_smem(L->r, M) > kMaxDecodeSmem) return NQ_ERR_SHAPE;
    if ((st = check_io(x, ybar, ws)) != NQ_OK) return st;
    if (!g_s1 || !g_s2) return NQ_ERR_NULL;
    if (!aligned16(g_s1) || !aligned16(g_s2)) return NQ_ERR_ALIGN;
    if (ws_bytes < nq_workspace_bytes(L, M)) return NQ_ERR_WORKSPACE;
    DeviceInfo* d = current_device();
    if (!d || !d->ok) return NQ_ERR_DEVICE;
    const nq_lrb_layer T = exchanged(L);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool pdl = pdl_enabled();
    // dL/ds1 from the layer with cotangent ybar; dL/ds2 from the exchanged layer, whose
    // intermediate is U^T (s1 . ybar), with cotangent x
    if (M <= NQ_MATVEC_MAX_M) {
        if ((st = nq_launch_decode(L, x, nullptr, M, ws, s, pdl, ybar, g_s1)) != NQ_OK) return st;
        return nq_launch_decode(&T, ybar, nullptr, M, ws, s, pdl, x, g_s2);
    }
    if ((st = nq_launch_prefill(L, x, nullptr, M, ws, s, pdl, ybar, g_s1)) != NQ_OK) return st;
    return nq_launch_prefill(&T, ybar, nullptr, M, ws, s, pdl, x, g_s2);
}

size_t nq_sign_grads_workspace_bytes(const nq_lrb_layer* L, int64_t M) {
    if (check_layer(L) != NQ_OK || M < 1) return 0;
    const nq_lrb_layer T = exchanged(L);
    return nq_sign_grads_ws(L, &T, M);
}

nq_status nq_lrb_sign_grads(const nq_lrb_layer* L, const uint16_t* x, const uint16_t* ybar, int64_t M, float* gU,
                            int64_t ldgu, float* gV, int64_t ldgv, void* ws, size_t ws_bytes, void* stream) {
    nq_status st = check_layer(L);
    if (st != NQ_OK) return st;
    if (M < 1) return NQ_ERR_SHAPE;
    if ((st = check_io(x, ybar, ws)) != NQ_OK) return st;
    if (!gU || !gV) return NQ_ERR_NULL;
    if (ldgu < L->r || ldgv < L->r) return NQ_ERR_SHAPE;
    if (!aligned16(gU) || !aligned16(gV) || (ldgu % 4) != 0 || (ldgv % 4) != 0) return NQ_ERR_ALIGN;
    const nq_lrb_layer T = exchanged(L);
    if (ws_bytes < nq_sign_grads_ws(L, &T, M)) return NQ_ERR_WORKSPACE;
    DeviceInfo* d = current_device();
    if (!d || !d->ok) return NQ_ERR_DEVICE;
    return nq_launch_sign_grads(L, &T, x, ybar, M, gU, ldgu, gV, ldgv, ws, static_cast<cudaStream_t>(stream),
                                pdl_enabled());
}

size_t nq_from_latent_workspace_bytes(int64_t d_out, int64_t d_in, int64_t r, int64_t ldu, int64_t ldv) {
    if (d_out < 1 || d_in < 1 || r < 32 || (r % 32) != 0 || r > NQ_MAX_RANK || ldu < r / 32 || ldv < r / 32) return 0;
    return nq_from_latent_ws(d_out, d_in, ldu, ldv);
}

nq_status nq_lrb_from_latent(const float* Uh, int64_t ld_uh, const float* Vh, int64_t ld_vh, int64_t d_out,
                             int64_t d_in, int64_t r, uint32_t* U, int64_t ldu, uint32_t* V, int64_t ldv,
                             uint16_t* s1, uint16_t* s2, double* eta, void* ws, size_t ws_bytes, void* stream) {
    if (d_out < 1 || d_in < 1 || r < 32 || (r % 32) != 0 || r > NQ_MAX_RANK) return NQ_ERR_SHAPE;
    if (ld_uh < r || ld_vh < r || ldu < r / 32 || ldv < r / 32) return NQ_ERR_SHAPE;
    if (!Uh || !Vh || !U || !V || !s1 || !s2 || !ws) return NQ_ERR_NULL;
    if (!aligned16(Uh) || !aligned16(Vh) || !aligned16(U) || !aligned16(V) || !aligned16(s1) || !aligned16(s2) ||
        !aligned16(ws) || (eta && (reinterpret_cast<uintptr_t>(eta) & 7u) != 0))
        return NQ_ERR_ALIGN;
    if (ws_bytes < nq_from_latent_ws(d_out, d_in, ldu, ldv)) return NQ_ERR_WORKSPACE;
    DeviceInfo* d = current_device();
    if (!d || !d->ok) return NQ_ERR_DEVICE;
    return nq_launch_from_latent(Uh, ld_uh, Vh, ld_vh, d_out, d_in, r, U, ldu, V, ldv, s1, s2, eta, ws,
                                 static_cast<cudaStream_t>(stream));
}

namespace {
// The unfused gate and up outputs ([M][d_out] bf16 each) follow the grouped workspace.
size_t mlp_tmp_offset(const nq_lrb_layer* const* gu, int64_t M) {
    return (nq_group_workspace_bytes(gu, 2, M) + 255) / 256 * 256;
}
size_t mlp_tmp_bytes(const nq_lrb_layer* gate, int64_t M) {
    return (static_cast<size_t>(M) * gate->d_out * 2 + 255) / 256 * 256;
}
}  // namespace

size_t nq_mlp_gate_up_workspace_bytes(const nq_lrb_layer* gate, const nq_lrb_layer* up, int64_t M) {
    if (M < 1 || check_layer(gate) != NQ_OK || check_layer(up) != NQ_OK) return 0;
    if (gate->d_in != up->d_in || gate->d_out != up->d_out) return 0;
    const nq_lrb_layer* gu[2] = {gate, up};
    return mlp_tmp_offset(gu, M) + 2 * mlp_tmp_bytes(gate, M);
}

nq_status nq_mlp_gate_up(const nq_lrb_layer* gate, const nq_lrb_layer* up, const uint16_t* x, uint16_t* h,
                         int64_t M, void* ws, size_t ws_bytes, void* stream) {
    nq_status st;
    if ((st = check_layer(gate)) != NQ_OK || (st = check_layer(up)) != NQ_OK) return st;
    if (M < 1 || gate->d_in != up->d_in || gate->d_out != up->d_out) return NQ_ERR_SHAPE;
    if (M <= NQ_MATVEC_MAX_M && (nq_decode_stage2_smem(gate->r, M) > kMaxDecodeSmem ||
                                 nq_decode_stage2_smem(up->r, M) > kMaxDecodeSmem))
        return NQ_ERR_SHAPE;
    if ((st = check_io(x, h, ws)) != NQ_OK) return st;
    if (ws_bytes < nq_mlp_gate_up_workspace_bytes(gate, up, M)) return NQ_ERR_WORKSPACE;
    DeviceInfo* d = current_device();
    if (!d || !d->ok) return NQ_ERR_DEVICE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M <= NQ_MATVEC_MAX_M && nq_decode_pair_smem(gate->r, up->r, M) <= kMaxDecodeSmem)
        return nq_launch_decode_gate_up(gate, up, x, h, M, ws, s, pdl_enabled());
    // unfused: both projections into the workspace, then SiLU.mul
    const nq_lrb_layer* gu[2] = {gate, up};
    char* tmp = static_cast<char*>(ws) + mlp_tmp_offset(gu, M);
    uint16_t* g = reinterpret_cast<uint16_t*>(tmp);
    uint16_t* u = reinterpret_cast<uint16_t*>(tmp + mlp_tmp_bytes(gate, M));
    uint16_t* outs[2] = {g, u};
    if (M <= NQ_MATVEC_MAX_M) {
        if ((st = nq_launch_decode_group(gu, 2, x, outs, M, ws, s, pdl_enabled())) != NQ_OK) return st;
    } else {
        for (int l = 0; l < 2; ++l)
            if ((st = nq_launch_prefill(gu[l], x, outs[l], M, ws, s, pdl_enabled())) != NQ_OK) return st;
    }
    return nq_launch_silu_mul(g, u, h, M * gate->d_out, s, pdl_enabled());
}

nq_status nq_silu_mul(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t n, void* stream) {
    if (n < 0) return NQ_ERR_SHAPE;
    if (n == 0) return NQ_OK;
    if (!g || !u || !h) return NQ_ERR_NULL;
    if (!aligned16(g) || !aligned16(u) || !aligned16(h)) return NQ_ERR_ALIGN;
    DeviceInfo* d = current_device();
    if (!d || !d->ok) return NQ_ERR_DEVICE;
    return nq_launch_silu_mul(g, u, h, n, static_cast<cudaStream_t>(stream), pdl_enabled());
}

nq_status nq_sync_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return NQ_ERR_LAUNCH;
    unsigned int word = 0u;
    if (cudaMemcpyFromSymbol(&word, nq::g_error_word, sizeof word) != cudaSuccess) return NQ_ERR_LAUNCH;
    if (word != 0u) {
        const unsigned int zero = 0u;
        cudaMemcpyToSymbol(nq::g_error_word, &zero, sizeof zero);
        if (word & nq::kErrTimeout) return NQ_ERR_TIMEOUT;
    }
    return NQ_OK;
}

}  // extern "C"
