// silu.cu -- h = bf16(silu(g) * u) between the gate/up and down projections of a Llama MLP
// block built from LRB layers.  Elementwise and HBM-bound: 16-byte vector loads/stores,
// fp32 math, CUDA's expf.
#include "nq_common.cuh"

namespace nq {

__device__ __forceinline__ uint16_t silu_mul1(uint16_t g, uint16_t u) {
    const float gf = bf16_bits_to_float(g);
    const float s = gf / (1.0f + expf(-gf));
    return float_to_bf16_bits(s * bf16_bits_to_float(u));
}

__global__ void __launch_bounds__(256) silu_mul_kernel(const uint16_t* __restrict__ g, const uint16_t* __restrict__ u,
                                                         uint16_t* __restrict__ h, int64_t n) {
    pdl_wait();
    const int64_t n8 = n / 8;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < n8; v += stride) {
        const uint4 gv = reinterpret_cast<const uint4*>(g)[v];
        const uint4 uv = reinterpret_cast<const uint4*>(u)[v];
        const uint32_t ga[4] = {gv.x, gv.y, gv.z, gv.w};
        const uint32_t ua[4] = {uv.x, uv.y, uv.z, uv.w};
        uint32_t ha[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint16_t lo = silu_mul1(static_cast<uint16_t>(ga[q] & 0xFFFFu), static_cast<uint16_t>(ua[q] & 0xFFFFu));
            const uint16_t hi = silu_mul1(static_cast<uint16_t>(ga[q] >> 16), static_cast<uint16_t>(ua[q] >> 16));
            ha[q] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
        }
        reinterpret_cast<uint4*>(h)[v] = make_uint4(ha[0], ha[1], ha[2], ha[3]);
    }
    // tail (n not a multiple of 8)
    for (int64_t e = n8 * 8 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += stride)
        h[e] = silu_mul1(g[e], u[e]);
}

}  // namespace nq

nq_status nq_launch_silu_mul(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t n, cudaStream_t stream,
                             bool pdl) {
    if (n == 0) return NQ_OK;
    int64_t blocks = (n / 8 + 255) / 256;
    if (blocks < 1) blocks = 1;
    const int64_t cap = static_cast<int64_t>(nq_host::sm_count()) * 4;
    if (blocks > cap) blocks = cap;
    void* args[] = {&g, &u, &h, &n};
    return nq_host::launch_pdl(reinterpret_cast<const void*>(nq::silu_mul_kernel), dim3(static_cast<unsigned>(blocks)),
                               dim3(256), 0, stream, args, pdl) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_LAUNCH;
}
