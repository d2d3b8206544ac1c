// noalloc.cu -- nq_lrb_matvec_noalloc: the decode path with its scratch in a fixed,
// statically sized device array owned by the library instead of a caller workspace.
//
// Who needs it: code that must not (or cannot) obtain device memory at the point where it
// runs a layer -- a plug-in inside an inference engine that hands it only its input and
// output tensors, code recorded while a stream is being captured into a CUDA graph (where
// cudaMalloc is not a stream operation and can implicitly synchronise the device), a
// latency-critical loop that cannot afford an allocator round trip, or a plain C caller
// with no allocator of its own.  Such callers still pass x and y; the intermediate t and the
// per-slice partials live in g_noalloc_scratch below.
#include <mutex>

#include "nq_common.cuh"

// Scratch shared by every call of nq_lrb_matvec_noalloc on a device.  Every GPU that loads
// the library holds this many bytes until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NQ_NOALLOC_SCRATCH_BYTES];

size_t nq_decode_workspace_bytes(int64_t d_in, int64_t r, int64_t M);
size_t nq_decode_stage2_smem(int64_t r, int64_t M);

namespace {

constexpr int kMaxDev = 64;

struct ScratchSlot {
    std::once_flag once;
    void* ptr = nullptr;  // device address of g_noalloc_scratch on this device
};
ScratchSlot g_slots[kMaxDev];

// Host code cannot use g_noalloc_scratch's name as a device address (it names a host-side
// shadow).  Its device address is queried once per device, with that device current.
void* scratch_address(int dev) {
    ScratchSlot* s = &g_slots[dev];
    std::call_once(s->once, [s]() {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess) s->ptr = p;
        else cudaGetLastError();
    });
    return s->ptr;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" NQ_API nq_status nq_lrb_matvec_noalloc(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M,
                                                  void* stream) {
    if (!L || !L->U || !L->V || !L->s1 || !L->s2 || !x || !y) return NQ_ERR_NULL;
    if (L->d_out <= 0 || L->d_in <= 0 || L->r <= 0 || (L->r % 32) != 0 || L->r > NQ_MAX_RANK_LIMIT) return NQ_ERR_SHAPE;
    if (L->ldu < L->r / 32 || L->ldv < L->r / 32) return NQ_ERR_SHAPE;
    if (M < 1 || M > NQ_MATVEC_MAX_M) return NQ_ERR_SHAPE;
    if (!aligned16(L->U) || !aligned16(L->V) || !aligned16(L->s1) || !aligned16(L->s2) || !aligned16(x) ||
        !aligned16(y))
        return NQ_ERR_ALIGN;
    if (nq_decode_workspace_bytes(L->d_in, L->r, M) > NQ_NOALLOC_SCRATCH_BYTES) return NQ_ERR_SCRATCH_LIMIT;
    if (nq_decode_stage2_smem(L->r, M) > 200 * 1024) return NQ_ERR_SHAPE;
    int dev = -1, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return NQ_ERR_DEVICE;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return NQ_ERR_DEVICE;
    void* scratch = scratch_address(dev);
    if (!scratch) return NQ_ERR_LAUNCH;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return nq_launch_decode(L, x, y, M, scratch, s, true);
}
