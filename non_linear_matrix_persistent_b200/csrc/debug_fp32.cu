// M²RNN debug mode: fp32 inputs, CUDA-core FFMA, accurate tanhf.
//
// A deliberately simple device implementation of the same recurrence
// (gist.science technical summary of "M²RNN: Non-Linear RNNs with
// Matrix-Valued States for Scalable Language Modeling", §2.1):
//   Z_t = tanh(H_{t-1} W + k_t v_tᵀ),  H_t = f_t H_{t-1} + (1 - f_t) Z_t,
//   y_t = H_tᵀ q_t (readout: this library's reading).
// One CTA per (b, h); the state lives in shared memory.  The backward
// recomputes the states of each chunk of C steps from the forward's
// checkpoints (the recompute strategy of the pages' §2.2) into a per-CTA
// workspace scratch and then walks the chunk in reverse.
#include "common.cuh"
#include "kernels.h"

namespace m2rnn {

constexpr int kDbgThreads = 256;

// One step of the recurrence for every element of the state owned by this
// thread: Hn = f·Hc + (1 - f)·tanh(Hc W + k vᵀ).  Hc, Hn are row-major K×V.
__device__ __forceinline__ void dbg_step(int K, int V, const float* Hc, const float* Ws, const float* kt,
                                         const float* vt, float ft, float* Hn) {
    for (int e = threadIdx.x; e < K * V; e += blockDim.x) {
        const int i = e / V, j = e % V;
        float acc = 0.f;
        for (int l = 0; l < V; ++l) acc = fmaf(Hc[i * V + l], Ws[l * V + j], acc);
        const float a = fmaf(kt[i], vt[j], acc);
        const float z = tanhf(a);
        Hn[e] = ft * Hc[e] + (1.f - ft) * z;
    }
}

__global__ void __launch_bounds__(kDbgThreads) m2rnn_fwd_fp32_kernel(const Params p) {
    extern __shared__ float sm[];
    const int K = p.K, V = p.V, T = p.T;
    const int bh = blockIdx.x, hd = bh % p.H;
    const int nck = (T + p.C - 1) / p.C;
    float* Ws = sm;
    float* Ha = Ws + V * V;
    float* Hb = Ha + K * V;
    float* kt = Hb + K * V;
    float* vt = kt + K;
    float* qt = vt + V;
    const float* Wg = static_cast<const float*>(p.W) + (size_t)hd * V * V;
    for (int e = threadIdx.x; e < V * V; e += blockDim.x) Ws[e] = Wg[e];
    const size_t sb = (size_t)bh * K * V;
    for (int e = threadIdx.x; e < K * V; e += blockDim.x) Ha[e] = p.H0 ? p.H0[sb + e] : 0.f;
    __syncthreads();
    if (p.ckpt)
        for (int e = threadIdx.x; e < K * V; e += blockDim.x) p.ckpt[(size_t)bh * nck * K * V + e] = Ha[e];
    float* Hc = Ha;
    float* Hn = Hb;
    const float* kg = static_cast<const float*>(p.k);
    const float* vg = static_cast<const float*>(p.v);
    const float* qg = static_cast<const float*>(p.q);
    const size_t qkb = (size_t)qk_pair(p, bh);   // k / q rows of this pair's head group
    for (int t = 0; t < T; ++t) {
        const size_t rk = (qkb * T + t) * K, rv = ((size_t)bh * T + t) * V;
        for (int i = threadIdx.x; i < K; i += blockDim.x) { kt[i] = kg[rk + i]; qt[i] = qg[rk + i]; }
        for (int j = threadIdx.x; j < V; j += blockDim.x) vt[j] = vg[rv + j];
        const float ft = gate_value(p, p.f[(size_t)bh * T + t]);
        __syncthreads();
        dbg_step(K, V, Hc, Ws, kt, vt, ft, Hn);
        __syncthreads();
        for (int j = threadIdx.x; j < V; j += blockDim.x) {
            float s = 0.f;
            for (int i = 0; i < K; ++i) s = fmaf(qt[i], Hn[i * V + j], s);
            p.y[rv + j] = s;
        }
        if (p.ckpt && (t + 1) < T && ((t + 1) % p.C) == 0)
            for (int e = threadIdx.x; e < K * V; e += blockDim.x)
                p.ckpt[((size_t)bh * nck + (t + 1) / p.C) * K * V + e] = Hn[e];
        float* tmp = Hc; Hc = Hn; Hn = tmp;
        __syncthreads();
    }
    if (p.HT)
        for (int e = threadIdx.x; e < K * V; e += blockDim.x) p.HT[sb + e] = Hc[e];
}

__device__ float block_sum(float v, float* red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float s = 0.f;
    for (int i = 0; i < nw; ++i) s += red[i];
    return s;
}

__global__ void __launch_bounds__(kDbgThreads) m2rnn_bwd_fp32_kernel(const Params p) {
    extern __shared__ float sm[];
    const int K = p.K, V = p.V, T = p.T, C = p.C;
    const int bh = blockIdx.x, hd = bh % p.H;
    const int nck = (T + C - 1) / C;
    float* Ws = sm;
    float* G = Ws + V * V;
    float* dA = G + K * V;
    float* kt = dA + K * V;
    float* vt = kt + K;
    float* qt = vt + V;
    float* dyt = qt + K;
    float* red = dyt + V;
    const float* Wg = static_cast<const float*>(p.W) + (size_t)hd * V * V;
    for (int e = threadIdx.x; e < V * V; e += blockDim.x) Ws[e] = Wg[e];
    const size_t sb = (size_t)bh * K * V;
    for (int e = threadIdx.x; e < K * V; e += blockDim.x) G[e] = p.dHT ? p.dHT[sb + e] : 0.f;
    float* dWp = p.dW_part + (size_t)bh * V * V;
    for (int e = threadIdx.x; e < V * V; e += blockDim.x) dWp[e] = 0.f;
    float* S = p.scratch + (size_t)bh * (C + 1) * K * V;   // states H_{c0} .. H_{c0+len}
    const float* kg = static_cast<const float*>(p.k);
    const float* vg = static_cast<const float*>(p.v);
    const float* qg = static_cast<const float*>(p.q);
    const float* dyg = static_cast<const float*>(p.dy);
    const size_t qkb = (size_t)qk_pair(p, bh);   // k / q rows of this pair's head group
    __syncthreads();
    for (int c = nck - 1; c >= 0; --c) {
        const int c0 = c * C, len = min(C, T - c0);
        const float* ck = p.ckpt + ((size_t)bh * nck + c) * K * V;
        for (int e = threadIdx.x; e < K * V; e += blockDim.x) S[e] = ck[e];
        __syncthreads();
        for (int u = 0; u < len; ++u) {   // recompute the chunk's states
            const int t = c0 + u;
            const size_t rq = (qkb * T + t) * K, rv = ((size_t)bh * T + t) * V;
            for (int i = threadIdx.x; i < K; i += blockDim.x) kt[i] = kg[rq + i];
            for (int j = threadIdx.x; j < V; j += blockDim.x) vt[j] = vg[rv + j];
            __syncthreads();
            dbg_step(K, V, S + (size_t)u * K * V, Ws, kt, vt, gate_value(p, p.f[(size_t)bh * T + t]),
                     S + (size_t)(u + 1) * K * V);
            __syncthreads();
        }
        for (int u = len - 1; u >= 0; --u) {
            const int t = c0 + u;
            const float* Hp = S + (size_t)u * K * V;
            const float* Hn = S + (size_t)(u + 1) * K * V;
            // rk: this pair's row of dk / dq (per head; summed over a head group afterwards)
            const size_t rk = ((size_t)bh * T + t) * K, rq = (qkb * T + t) * K, rv = ((size_t)bh * T + t) * V;
            for (int i = threadIdx.x; i < K; i += blockDim.x) { kt[i] = kg[rq + i]; qt[i] = qg[rq + i]; }
            for (int j = threadIdx.x; j < V; j += blockDim.x) { vt[j] = vg[rv + j]; dyt[j] = dyg[rv + j]; }
            const float ft = gate_value(p, p.f[(size_t)bh * T + t]);
            __syncthreads();
            for (int e = threadIdx.x; e < K * V; e += blockDim.x) G[e] = fmaf(qt[e / V], dyt[e % V], G[e]);
            __syncthreads();
            float dfp = 0.f;
            for (int e = threadIdx.x; e < K * V; e += blockDim.x) {
                const int i = e / V, j = e % V;
                float acc = 0.f;
                for (int l = 0; l < V; ++l) acc = fmaf(Hp[i * V + l], Ws[l * V + j], acc);
                const float z = tanhf(fmaf(kt[i], vt[j], acc));
                dfp = fmaf(G[e], Hp[e] - z, dfp);
                dA[e] = (1.f - ft) * G[e] * (1.f - z * z);
            }
            const float dfs = block_sum(dfp, red);
            if (threadIdx.x == 0) p.df[(size_t)bh * T + t] = gate_grad(p, p.f[(size_t)bh * T + t], dfs);
            __syncthreads();
            for (int i = threadIdx.x; i < K; i += blockDim.x) {
                float s = 0.f, s2 = 0.f;
                for (int j = 0; j < V; ++j) {
                    s = fmaf(dA[i * V + j], vt[j], s);
                    s2 = fmaf(Hn[i * V + j], dyt[j], s2);
                }
                p.dk[rk + i] = s;
                p.dq[rk + i] = s2;
            }
            for (int j = threadIdx.x; j < V; j += blockDim.x) {
                float s = 0.f;
                for (int i = 0; i < K; ++i) s = fmaf(dA[i * V + j], kt[i], s);
                p.dv[rv + j] = s;
            }
            for (int e = threadIdx.x; e < V * V; e += blockDim.x) {
                const int l = e / V, j = e % V;
                float s = 0.f;
                for (int i = 0; i < K; ++i) s = fmaf(Hp[i * V + l], dA[i * V + j], s);
                dWp[e] += s;
            }
            for (int e = threadIdx.x; e < K * V; e += blockDim.x) {
                const int i = e / V, l = e % V;
                float s = 0.f;
                for (int j = 0; j < V; ++j) s = fmaf(dA[i * V + j], Ws[l * V + j], s);
                G[e] = fmaf(ft, G[e], s);
            }
            __syncthreads();
        }
    }
    for (int e = threadIdx.x; e < K * V; e += blockDim.x) p.dH0[sb + e] = G[e];
}

__global__ void m2rnn_dw_reduce_kernel(const Params p) {
    const size_t VV = (size_t)p.V * p.V;
    const size_t n = (size_t)p.H * VV;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const size_t h = e / VV, r = e % VV;
        float s = 0.f;
        for (int b = 0; b < p.B; ++b)
            for (int sl = 0; sl < p.dw_parts; ++sl) s += p.dW_part[(((size_t)b * p.H + h) * p.dw_parts + sl) * VV + r];
        p.dW[e] = s;
    }
}

cudaError_t launch_fwd_fp32(const Params& p, cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)p.V * p.V + 2 * (size_t)p.K * p.V + 2 * p.K + p.V);
    cudaError_t e = cudaFuncSetAttribute(m2rnn_fwd_fp32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    m2rnn_fwd_fp32_kernel<<<p.B * p.H, kDbgThreads, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_dw_reduce(const Params& p, cudaStream_t s) {
    const size_t n = (size_t)p.H * p.V * p.V;
    const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
    m2rnn_dw_reduce_kernel<<<blocks, 256, 0, s>>>(p);
    return cudaGetLastError();
}

size_t bwd_fp32_workspace(int B, int H, int K, int V, int C) {
    return sizeof(float) * ((size_t)B * H * V * V + (size_t)B * H * (C + 1) * K * V);
}

cudaError_t launch_bwd_fp32(const Params& p, cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)p.V * p.V + 2 * (size_t)p.K * p.V + 2 * p.K + 2 * p.V + 32);
    cudaError_t e = cudaFuncSetAttribute(m2rnn_bwd_fp32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    m2rnn_bwd_fp32_kernel<<<p.B * p.H, kDbgThreads, smem, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_dw_reduce(p, s);
}

}  // namespace m2rnn
