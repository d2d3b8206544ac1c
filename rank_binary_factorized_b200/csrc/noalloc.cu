// noalloc.cu -- nq_lrb_matvec_noalloc: the decode path with its scratch in a fixed,
// statically sized device array owned by the library instead of a caller workspace.
//
// Who needs it: code that must not (or cannot) obtain device memory at the point where it
// runs a layer -- a plug-in inside an inference engine that hands it only its input and
// output tensors, a latency-critical loop that cannot afford an allocator round trip, or a
// plain C caller with no allocator of its own.  Such callers still pass x and y; the
// intermediate t and the per-slice partials live in g_noalloc_scratch below.
#include <atomic>

#include "nq_common.cuh"

// Scratch shared by every call of nq_lrb_matvec_noalloc on a device.  Every GPU that loads
// the library holds this many bytes until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NQ_NOALLOC_SCRATCH_BYTES];

size_t nq_decode_workspace_bytes(int64_t d_in, int64_t r, int64_t M);

namespace {

constexpr int kMaxDev = 64;

// Device address of g_noalloc_scratch per device; null until a lookup has succeeded.  Host
// code cannot use the array's name as a device address (it names a host-side shadow), so the
// address is queried with the device current.  A failed lookup is not remembered: the next
// call tries again.
std::atomic<void*> g_scratch[kMaxDev];

void* scratch_address(int dev) {
    void* p = g_scratch[dev].load(std::memory_order_acquire);
    if (p) return p;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();  // leave no sticky error behind for the caller
        return nullptr;
    }
    g_scratch[dev].store(p, std::memory_order_release);  // racing threads store the same value
    return p;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" NQ_API nq_status nq_lrb_matvec_noalloc(const nq_lrb_layer* L, const uint16_t* x, uint16_t* y, int64_t M,
                                                  void* stream) {
    // the same checks as nq_lrb_matvec, in the same order
    nq_status st = nq_host::check_decode_call(L, M);
    if (st != NQ_OK) return st;
    if (!x || !y) return NQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(y)) return NQ_ERR_ALIGN;
    if (nq_decode_workspace_bytes(L->d_in, L->r, M) > NQ_NOALLOC_SCRATCH_BYTES) return NQ_ERR_SCRATCH_LIMIT;
    if (!nq_host::device_ready()) return NQ_ERR_DEVICE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return NQ_ERR_DEVICE;
    void* scratch = scratch_address(dev);
    if (!scratch) return NQ_ERR_LAUNCH;
    return nq_launch_decode(L, x, y, M, scratch, static_cast<cudaStream_t>(stream), nq_host::pdl_on());
}
