// M²RNN forward scan for few (b, h) pairs: two state rows per warp, CUDA-core
// FFMA, no per-step barrier.
//
// Recurrence (gist.science technical summary of "M²RNN: Non-Linear RNNs with
// Matrix-Valued States for Scalable Language Modeling", §2.1):
//   Z_t = tanh(H_{t-1} W + k_t v_tᵀ),  H_t = f_t H_{t-1} + (1 - f_t) Z_t,
// plus the readout y_t = H_tᵀ q_t (this library's reading).  Row i of H_t
// depends only on row i of H_{t-1}, on W and on the step's inputs:
//   h_t = f_t h_{t-1} + (1 - f_t) tanh(h_{t-1} W + k_t[i] v_t),
// so the rows of a pair are independent recurrences that share W and v_t.
// The pages parallelise over batch × head with one matrix state per SM
// (§2.2).  With few pairs that leaves most of the GPU idle, and the
// tensor-core kernel's step is bound by its MMA round trip (issue, commit,
// barrier wake-up: ~1,000 cycles), not by arithmetic.  This kernel gives each
// warp two state rows for all T steps instead, with W resident in registers,
// so a step needs no block-level synchronisation at all: the warp shares its
// two rows through shared memory (__syncwarp), every lane reads both rows in
// 16-byte broadcast loads, and lane l forms columns 2l and 2l + 1 of each
// row's product h_{t-1}·W with packed FFMA2 (W[l'][2l], W[l'][2l + 1] as fp32
// pairs, 64 of them, shared by the two rows) in four accumulator chains per
// row; a lane's two adjacent columns move in 8-byte accesses.
// Measured on B200 at the long B = 1 workload (1,024 rows on 128 SMs): one
// row per warp 8.1 ms, two rows per warp 6.2 ms (4.8 ms with the step loop
// below); slower were the same with the h row stored as duplicated pairs
// (7.9 ms), a row pair split over two warps by columns (8.5 ms) and a
// two-dimensional split of the product over the lanes with a shuffle
// reduce-scatter (8.1 / 8.7 ms).
//
// Arithmetic: fp32 products of the fp32 state with W (bf16 values, exact in
// fp32), fp32 sums in a fixed order, the exp-based tanh of the tensor-core
// kernels (here on packed pairs, tanh2_ex2, same bits; in the instantiation
// that writes the backward's checkpoints tanh2_acc, which keeps its relative
// accuracy near zero; tanh.approx.f32 in the fast-tanh mode), the blend
// h + (1 - f)(z - h).  This is more precise than the tensor-core kernel's
// compensated bf16 operand, so the two kernels' states agree to rounding, not
// bit for bit; within this kernel a row's result does not depend on the rest
// of the batch or on how rows are grouped into CTAs.
//
// Layout: one CTA per (b, h) and slice of RS = 8 rows (4 row warps), plus a
// bulk-copy producer warp (this slice's 8 values of k_t and q_t, the pair's
// v_t, f_t for TC steps per ring stage) and a storer warp that sums the row
// warps' readout partials (each warp's two rows q_t[i]·h_t[i, :] +
// q_t[i+1]·h_t[i+1, :]) in warp order.  With several slices per
// pair the slices' partial readouts go to the workspace and
// m2rnn_y_reduce_kernel adds them in slice order.  Supported: V = 64 (W takes
// 128 registers per lane) and at most 148 CTAs (one wave, one CTA per SM).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace m2rnn {

template <int RS_>
struct FwdRowsCfg {
    static constexpr int V = 64;
    static constexpr int RS = RS_;                 // rows per CTA
    static constexpr int RW = 2;                   // rows per warp (sharing the W registers)
    static constexpr int NWR = RS / RW;            // row warps
    static constexpr int TC = 16;                  // steps per ring stage
    static constexpr int S = 4;                    // ring stages
    static constexpr int W_PROD = NWR, W_STORE = NWR + 1;
    static constexpr int NTHREADS = (NWR + 2) * 32;
    static constexpr int ST_K = 0;                 // [TC][RS] bf16
    static constexpr int ST_Q = TC * RS * 2;       // [TC][RS] bf16
    static constexpr int ST_V = 2 * TC * RS * 2;   // [TC][V] bf16
    static constexpr int ST_F = ST_V + TC * V * 2; // [TC] fp32
    static constexpr int STAGE_BYTES = ((ST_F + TC * 4) + 127) / 128 * 128;
    static constexpr int YBUF_BYTES = TC * NWR * V * 4;  // [TC][NWR][V] readout partials, one per row warp
    static constexpr int HROW_BYTES = 2 * RW * V * 4;    // per warp: its rows, double-buffered
    static constexpr int OFF_RING = 0;
    static constexpr int OFF_Y = OFF_RING + S * STAGE_BYTES;
    static constexpr int OFF_H = OFF_Y + 2 * YBUF_BYTES;
    static constexpr int OFF_BAR = OFF_H + NWR * HROW_BYTES;
    static constexpr int NBAR = 2 * S + 4;         // in_full, in_empty, ypfull[2], ypempty[2]
    static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16;
    static_assert(RS == 8, "rows per CTA: the per-step k / q copies are RS·2 = 16 bytes");
    static_assert(STAGE_BYTES % 128 == 0 && OFF_Y % 16 == 0 && OFF_H % 16 == 0 && OFF_BAR % 8 == 0, "alignment");
    static_assert(SMEM_BYTES <= 227 * 1024, "smem");
};

// CKPT: the call writes checkpoints (p.ckpt != nullptr); without them the
// kernel carries no checkpoint code (a per-step test of the next checkpoint
// step measured 3% slower at the long B = 1 workload).
template <int RS, bool FAST, bool CKPT>
__global__ void __launch_bounds__(FwdRowsCfg<RS>::NTHREADS, 1) m2rnn_fwd_rows_kernel(const Params p) {
    using C = FwdRowsCfg<RS>;
    constexpr int V = C::V;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nsl = p.slices;
    const int bh = blockIdx.x / nsl, sl = blockIdx.x % nsl;
    const int K = p.K, koff = sl * RS;
    const int hd = bh % p.H;
    const int T = p.T;
    const int nchunks = (T + C::TC - 1) / C::TC;
    const int nck = (T + p.C - 1) / p.C;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    auto in_full = [&](int s) { return bar(s); };
    auto in_empty = [&](int s) { return bar(C::S + s); };
    auto ypfull = [&](int i) { return bar(2 * C::S + i); };
    auto ypempty = [&](int i) { return bar(2 * C::S + 2 + i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + C::NBAR);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::S; ++s) {
            mbar_init(in_full(s), 1);
            mbar_init(in_empty(s), C::NWR);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(ypfull(i), C::NWR);
            mbar_init(ypempty(i), 1);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();

    if (warp < C::NWR) {
        // ------------------------------------------------------------ two state rows per warp
        const int r0 = warp * 2;                   // first row of this warp within the slice
        const int i = koff + r0;                   // its state row
        const int j0 = 2 * lane;                   // state columns j0, j0 + 1 of this lane (8-byte accesses)
        // W columns j0, j0 + 1 as fp32 pairs, resident for all T steps
        float2 Wr[V];
        {
            const uint16_t* Wg = static_cast<const uint16_t*>(p.W) + (size_t)hd * V * V;
#pragma unroll
            for (int l = 0; l < V; ++l) {
                const uint32_t w2 = *reinterpret_cast<const uint32_t*>(Wg + l * V + j0);
                Wr[l] = make_float2(bf16lo_to_f32(w2), bf16hi_to_f32(w2));
            }
        }
        const size_t srow0 = ((size_t)bh * K + i) * V, srow1 = srow0 + V;
        float2 h0 = p.H0 != nullptr ? *reinterpret_cast<const float2*>(p.H0 + srow0 + j0) : make_float2(0.f, 0.f);
        float2 h1 = p.H0 != nullptr ? *reinterpret_cast<const float2*>(p.H0 + srow1 + j0) : make_float2(0.f, 0.f);
        if (CKPT) {
            float* ck = p.ckpt + (size_t)bh * nck * K * V + (size_t)i * V;
            *reinterpret_cast<float2*>(ck + j0) = h0;
            *reinterpret_cast<float2*>(ck + V + j0) = h1;
        }
        float* hrow = reinterpret_cast<float*>(smem + C::OFF_H + warp * C::HROW_BYTES);
        // next checkpoint step as a running count (no per-step remainder by the run-time stride)
        int ck_next = p.C, ck_idx = 0;
        bool ok = true;
        // one chunk of TC steps per outer iteration: the ring and readout waits and
        // arrivals stay out of the step loop, whose body is then one straight
        // block (with the waits inside it, under a per-step test, the scan took
        // 5.97 instead of 5.01 ms at the long B = 1 workload), unrolled by 4
        // (5.01 -> 4.83 ms; by 8 or 16, 5.07 and 5.93 ms)
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c % C::S, nt = min(C::TC, T - c * C::TC);
            const uint8_t* st = smem + C::OFF_RING + s * C::STAGE_BYTES;
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(in_full(s), (c / C::S) & 1, abort_flag, p));
            if (ok && c >= 2)
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(ypempty(c & 1), ((c >> 1) - 1) & 1, abort_flag, p));
            if (!ok) break;
#pragma unroll 4
            for (int tt = 0; tt < nt; ++tt) {
                const int t = c * C::TC + tt;
                // both rows of h_{t-1} to every lane.  The buffer alternates by step:
                // every lane read this one at step t-2 before it reached the
                // __syncwarp of step t-1, which this lane has passed.
                float* hb = hrow + (t & 1) * 2 * V;
                *reinterpret_cast<float2*>(hb + j0) = h0;
                *reinterpret_cast<float2*>(hb + V + j0) = h1;
                __syncwarp();
                const uint32_t kk = *reinterpret_cast<const uint32_t*>(st + C::ST_K + (tt * RS + r0) * 2);
                const uint16_t* vt = reinterpret_cast<const uint16_t*>(st + C::ST_V + tt * V * 2);
                const uint32_t vv = *reinterpret_cast<const uint32_t*>(vt + j0);
                const float2 v2 = make_float2(bf16lo_to_f32(vv), bf16hi_to_f32(vv));
                // h_{t-1}·W[:, (j0, j0 + 1)] for both rows: four accumulator chains per row over l mod 4
                float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0, b0 = a0, b1 = a0, b2 = a0, b3 = a0;
                const float4* hb4 = reinterpret_cast<const float4*>(hb);
    #pragma unroll
                for (int b = 0; b < V / 4; b += 4) {
                    float4 xs[4], ys[4];
    #pragma unroll
                    for (int u = 0; u < 4; ++u) { xs[u] = hb4[b + u]; ys[u] = hb4[V / 4 + b + u]; }
    #pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int l4 = b + u;
                        a0 = __ffma2_rn(make_float2(xs[u].x, xs[u].x), Wr[4 * l4], a0);
                        b0 = __ffma2_rn(make_float2(ys[u].x, ys[u].x), Wr[4 * l4], b0);
                        a1 = __ffma2_rn(make_float2(xs[u].y, xs[u].y), Wr[4 * l4 + 1], a1);
                        b1 = __ffma2_rn(make_float2(ys[u].y, ys[u].y), Wr[4 * l4 + 1], b1);
                        a2 = __ffma2_rn(make_float2(xs[u].z, xs[u].z), Wr[4 * l4 + 2], a2);
                        b2 = __ffma2_rn(make_float2(ys[u].z, ys[u].z), Wr[4 * l4 + 2], b2);
                        a3 = __ffma2_rn(make_float2(xs[u].w, xs[u].w), Wr[4 * l4 + 3], a3);
                        b3 = __ffma2_rn(make_float2(ys[u].w, ys[u].w), Wr[4 * l4 + 3], b3);
                    }
                }
                float2 A0 = __fadd2_rn(__fadd2_rn(a0, a1), __fadd2_rn(a2, a3));
                float2 A1 = __fadd2_rn(__fadd2_rn(b0, b1), __fadd2_rn(b2, b3));
                const float k0 = bf16lo_to_f32(kk), k1 = bf16hi_to_f32(kk);
                A0 = __ffma2_rn(make_float2(k0, k0), v2, A0);
                A1 = __ffma2_rn(make_float2(k1, k1), v2, A1);
                const float g = 1.f - *reinterpret_cast<const float*>(st + C::ST_F + tt * 4);
                {
                    const float2 z01 = FAST   ? make_float2(tanh_approx(A0.x), tanh_approx(A0.y))
                                      : CKPT ? tanh2_acc(A0) : tanh2_ex2(A0);
                    const float2 z23 = FAST   ? make_float2(tanh_approx(A1.x), tanh_approx(A1.y))
                                      : CKPT ? tanh2_acc(A1) : tanh2_ex2(A1);
                    h0 = __ffma2_rn(make_float2(g, g), __fadd2_rn(z01, make_float2(-h0.x, -h0.y)), h0);
                    h1 = __ffma2_rn(make_float2(g, g), __fadd2_rn(z23, make_float2(-h1.x, -h1.y)), h1);
                }
                // readout partials of the two rows: q_t[i]·h_t[i, :]
                const uint32_t qq = *reinterpret_cast<const uint32_t*>(st + C::ST_Q + (tt * RS + r0) * 2);
                const float q0 = bf16lo_to_f32(qq), q1 = bf16hi_to_f32(qq);
                // the warp's two rows summed here, so that the storer adds NWR partials
                float* yb = reinterpret_cast<float*>(smem + C::OFF_Y + (c & 1) * C::YBUF_BYTES) + (tt * C::NWR + warp) * V;
                *reinterpret_cast<float2*>(yb + j0) = make_float2(fmaf(q1, h1.x, q0 * h0.x), fmaf(q1, h1.y, q0 * h0.y));
                if (CKPT && t + 1 == ck_next) {   // checkpoint ck_idx = H_{t+1}
                    ck_next += p.C;
                    ++ck_idx;
                    if ((t + 1) < T) {
                        float* ck = p.ckpt + ((size_t)bh * nck + ck_idx) * K * V + (size_t)i * V;
                        *reinterpret_cast<float2*>(ck + j0) = h0;
                        *reinterpret_cast<float2*>(ck + V + j0) = h1;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(in_empty(s));
                mbar_arrive(ypfull(c & 1));
            }
        }
        if (ok && p.HT != nullptr) {
            *reinterpret_cast<float2*>(p.HT + srow0 + j0) = h0;
            *reinterpret_cast<float2*>(p.HT + srow1 + j0) = h1;
        }
    } else if (warp == C::W_PROD) {
        // ------------------------------------------------------------ producer
        const int qkb = qk_pair(p, bh);   // k / q rows of this pair's head group
        int last = -1;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % C::S;
            if (p.fault == 1 && c >= 1) break;   // injected: stop feeding the ring after the first chunk
            if (c >= C::S) {
                const bool ok =
                    __all_sync(0xffffffffu, mbar_wait_bounded(in_empty(s), ((c / C::S) - 1) & 1, abort_flag, p));
                if (!ok) break;
            }
            const int t0 = c * C::TC, nt = min(C::TC, T - t0);
            uint8_t* st = smem + C::OFF_RING + s * C::STAGE_BYTES;
            if (lane < nt)
                reinterpret_cast<float*>(st + C::ST_F)[lane] = gate_value(p, p.f[(size_t)bh * T + t0 + lane]);
            __syncwarp();
            if (lane == 0) {
                const uint32_t vb = (uint32_t)(nt * V * 2);
                mbar_arrive_expect_tx(in_full(s), (uint32_t)(2 * nt * RS * 2) + vb);
                bulk_g2s(smem_u32(st + C::ST_V), static_cast<const uint16_t*>(p.v) + ((size_t)bh * T + t0) * V, vb,
                         in_full(s));
            }
            __syncwarp();
            if (lane < nt) {   // this slice's RS values of each step's k and q row
                const size_t r = ((size_t)qkb * T + t0 + lane) * K + koff;
                bulk_g2s(smem_u32(st + C::ST_K + lane * RS * 2), static_cast<const uint16_t*>(p.k) + r, RS * 2,
                         in_full(s));
                bulk_g2s(smem_u32(st + C::ST_Q + lane * RS * 2), static_cast<const uint16_t*>(p.q) + r, RS * 2,
                         in_full(s));
            }
            last = c;
        }
        // copies still in flight must land before the CTA exits
        if (lane == 0)
            for (int c = max(0, last - C::S + 1); c <= last; ++c) mbar_wait_drain(in_full(c % C::S), (c / C::S) & 1, p);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ y storer
        float* yout = nsl == 1 ? p.y : p.ypart + (size_t)sl * p.B * p.H * T * V;
        for (int c = 0; c < nchunks; ++c) {
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(ypfull(c & 1), (c >> 1) & 1, abort_flag, p));
            if (!ok) break;
            const int t0 = c * C::TC, nt = min(C::TC, T - t0);
            const float* yb = reinterpret_cast<const float*>(smem + C::OFF_Y + (c & 1) * C::YBUF_BYTES);
            float* yg = yout + ((size_t)bh * T + t0) * V;
            for (int e = lane * 4; e < nt * V; e += 128) {
                const int tt = e / V, jj = e % V;
                const float* src = yb + tt * C::NWR * V + jj;
                float4 a = *reinterpret_cast<const float4*>(src);
#pragma unroll
                for (int r = 1; r < C::NWR; ++r) {
                    const float4 b = *reinterpret_cast<const float4*>(src + r * V);
                    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
                }
                *reinterpret_cast<float4*>(yg + e) = a;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(ypempty(c & 1));
        }
    }
}

// Rows per CTA of the row kernel for B·H pairs of K x V states, or 0 when the
// tensor-core kernel takes the problem: V = 64 and few enough rows that every
// row gets a warp, 8 rows per CTA and one CTA per SM.
int fwd_rows_per_cta(int B, int H, int K, int V) {
    const long long pairs = (long long)B * H;
    return (V == 64 && K % 8 == 0 && pairs * (K / 8) <= kNumSMs) ? 8 : 0;
}

template <int RS>
static cudaError_t launch_rows(const Params& p0, cudaStream_t stream) {
    using C = FwdRowsCfg<RS>;
    Params p = p0;
    p.slices = p.K / RS;
    auto kern = p.ckpt != nullptr
                    ? (p.fast_tanh ? m2rnn_fwd_rows_kernel<RS, true, true> : m2rnn_fwd_rows_kernel<RS, false, true>)
                    : (p.fast_tanh ? m2rnn_fwd_rows_kernel<RS, true, false> : m2rnn_fwd_rows_kernel<RS, false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<p.B * p.H * p.slices, C::NTHREADS, C::SMEM_BYTES, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.slices == 1) return e;
    return launch_y_reduce(p, stream);
}

cudaError_t launch_fwd_rows(const Params& p, cudaStream_t s) {
    if (fwd_rows_per_cta(p.B, p.H, p.K, p.V) == 8) return launch_rows<8>(p, s);
    return cudaErrorNotSupported;
}

}  // namespace m2rnn
