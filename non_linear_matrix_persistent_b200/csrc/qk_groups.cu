// Sum of per-head dk / dq over the heads of a k / q group (grouped k and q:
// head h of H uses group h / (H/G)).  The backward kernels write one dk and
// one dq row per (b, h, t); a shared input's gradient is the sum of its uses'.
#include "kernels.h"

namespace m2rnn {

// dk[b, g] = sum_{j < H/G} dk_part[b, g·(H/G) + j] in ascending j, and the
// same for dq.  Rows of T·K fp32 (T·K is a multiple of 4: K is a multiple of
// 16), read and written as float4; the grid strides over both outputs.
__global__ void m2rnn_qk_group_reduce_kernel(const float4* __restrict__ dk_part, const float4* __restrict__ dq_part,
                                             float4* __restrict__ dk, float4* __restrict__ dq, int B, int H, int G,
                                             size_t tk4) {
    const size_t per = (size_t)G * tk4, n = (size_t)B * per;
    const int hpg = H / G;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < 2 * n; e += (size_t)gridDim.x * blockDim.x) {
        const bool second = e >= n;
        const size_t o = second ? e - n : e;
        const size_t b = o / per, rem = o % per, g = rem / tk4, r = rem % tk4;
        const float4* src = (second ? dq_part : dk_part) + (b * H + g * hpg) * tk4 + r;
        float4 s = src[0];
        for (int j = 1; j < hpg; ++j) {
            const float4 x = src[(size_t)j * tk4];
            s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
        }
        (second ? dq : dk)[o] = s;
    }
}

cudaError_t launch_qk_group_reduce(const Params& p, const float* dk_part, const float* dq_part, float* dk, float* dq,
                                   cudaStream_t s) {
    const size_t tk4 = (size_t)p.T * p.K / 4;
    const size_t n = 2 * (size_t)p.B * p.G * tk4;
    if (n == 0) return cudaSuccess;
    const size_t want = (n + 255) / 256, cap = (size_t)kNumSMs * 8;
    m2rnn_qk_group_reduce_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, s>>>(
        reinterpret_cast<const float4*>(dk_part), reinterpret_cast<const float4*>(dq_part),
        reinterpret_cast<float4*>(dk), reinterpret_cast<float4*>(dq), p.B, p.H, p.G, tk4);
    return cudaGetLastError();
}

}  // namespace m2rnn
