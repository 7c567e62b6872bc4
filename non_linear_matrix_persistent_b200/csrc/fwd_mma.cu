// M²RNN forward scan with the state resident in registers (mma.sync).
//
// Same recurrence and readout as the tcgen05 forward (gist.science summary of
// "M²RNN", §2.1: Z_t = tanh(H_{t-1} W + k_t v_tᵀ), H_t = f_t H_{t-1} +
// (1 - f_t) Z_t; y_t = H_tᵀ q_t), as a latency-oriented alternative for
// V = 64, K <= 64.  Rows of H are independent given W, v_t and f_t, so each
// warp owns 16 rows for all T steps and never waits for another warp inside
// a step: H_{t-1} W is sixty-four m16n8k16 warp MMAs (4 k-steps × 8 column
// tiles × the hi and lo halves of the compensated bf16 operand) with W held
// as B fragments in registers, and the fp32 accumulator layout of one step is
// the A-operand layout of the next (rows g and g+8, column pairs 2t, 2t+1),
// so the state never leaves the registers.  There is no tensor memory, no
// shared-memory operand and no barrier per step; warps meet only at the
// 16-step input stages and the readout buffer.
//
// Warps: [0, K/16) compute, then one bulk-copy producer (k, q, v, f for 16
// steps per stage) and one storer that sums the warps' readout partials.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace m2rnn {

template <int K_>
struct FwdMmaCfg {
    static constexpr int K = K_, V = 64;
    static constexpr int NW = K / 16;          // compute warps, 16 rows each
    static constexpr int NT8 = V / 8;          // column tiles of 8
    static constexpr int KSTEPS = V / 16;      // k-steps of 16
    static constexpr int TC = 16;              // steps per ring stage
    static constexpr int S = 4;                // ring stages
    static constexpr int W_PROD = NW, W_STORE = NW + 1;
    static constexpr int NTHREADS = (NW + 2) * 32;
    static constexpr int ST_K = 0;
    static constexpr int ST_Q = TC * K * 2;
    static constexpr int ST_V = 2 * TC * K * 2;
    static constexpr int ST_F = ST_V + TC * V * 2;
    static constexpr int STAGE_BYTES = ((ST_F + TC * 4) + 127) / 128 * 128;
    static constexpr int YBUF_BYTES = NW * TC * V * 4;   // one partial readout per warp
    static constexpr int OFF_RING = 0;
    static constexpr int OFF_Y = OFF_RING + S * STAGE_BYTES;
    static constexpr int OFF_BAR = OFF_Y + 2 * YBUF_BYTES;
    static constexpr int NBAR = 2 * S + 4;
    static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16;
    static_assert(K == 16 || K == 32 || K == 64, "K");
};

// D (+)= A · B, m16n8k16, bf16 inputs, fp32 accumulator.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int K>
__global__ void __launch_bounds__(FwdMmaCfg<K>::NTHREADS, 1) m2rnn_fwd_mma_kernel(const Params p) {
    using C = FwdMmaCfg<K>;
    constexpr int V = C::V;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x, hd = bh % p.H;
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
            mbar_init(in_empty(s), C::NW);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(ypfull(i), C::NW);
            mbar_init(ypempty(i), 1);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();

    if (warp < C::NW) {
        // ------------------------------------------------------------ compute warp: rows 16w .. 16w+15
        const int g = lane >> 2, tq = lane & 3;
        const int i0 = 16 * warp + g, i1 = i0 + 8;   // this thread's two rows
        const size_t sbase = (size_t)bh * K * V;
        // W as B fragments: k = rows l of W, n = columns j; element pairs along k
        uint32_t wb[C::KSTEPS][C::NT8][2];
        {
            const uint16_t* Wg = static_cast<const uint16_t*>(p.W) + (size_t)hd * V * V;
#pragma unroll
            for (int ks = 0; ks < C::KSTEPS; ++ks)
#pragma unroll
                for (int nt = 0; nt < C::NT8; ++nt)
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb) {
                        const int l = 16 * ks + 2 * tq + 8 * hb, jj = 8 * nt + g;
                        wb[ks][nt][hb] = (uint32_t)Wg[l * V + jj] | ((uint32_t)Wg[(l + 1) * V + jj] << 16);
                    }
        }
        // state in the accumulator layout: h[nt] = (i0, c), (i0, c+1), (i1, c), (i1, c+1), c = 8nt + 2tq
        float h[C::NT8][4];
#pragma unroll
        for (int nt = 0; nt < C::NT8; ++nt) {
            const int c0 = 8 * nt + 2 * tq;
            if (p.H0 != nullptr) {
                const float2 a = *reinterpret_cast<const float2*>(p.H0 + sbase + (size_t)i0 * V + c0);
                const float2 b = *reinterpret_cast<const float2*>(p.H0 + sbase + (size_t)i1 * V + c0);
                h[nt][0] = a.x; h[nt][1] = a.y; h[nt][2] = b.x; h[nt][3] = b.y;
            } else {
                h[nt][0] = h[nt][1] = h[nt][2] = h[nt][3] = 0.f;
            }
        }
        auto store_state = [&](float* dst) {   // [K][V] fp32, this thread's 32 values
#pragma unroll
            for (int nt = 0; nt < C::NT8; ++nt) {
                const int c0 = 8 * nt + 2 * tq;
                *reinterpret_cast<float2*>(dst + (size_t)i0 * V + c0) = make_float2(h[nt][0], h[nt][1]);
                *reinterpret_cast<float2*>(dst + (size_t)i1 * V + c0) = make_float2(h[nt][2], h[nt][3]);
            }
        };
        if (p.ckpt != nullptr) store_state(p.ckpt + (size_t)bh * nck * K * V);
        // next checkpoint step as a running count (no per-step remainder by the run-time stride)
        int ck_next = p.ckpt != nullptr ? p.C : T + 1, ck_idx = 0;

        bool ok = true;
        // one chunk of TC steps per outer iteration: the ring and readout waits
        // and arrivals stay out of the step loop, whose body is one straight block
        // (1.73 -> 1.57 ms at the 410M layer), unrolled by 2 (1.56 ms; by 4, 2.11)
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c % C::S, nt = min(C::TC, T - c * C::TC);
            const uint8_t* st = smem + C::OFF_RING + s * C::STAGE_BYTES;
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(in_full(s), (c / C::S) & 1, abort_flag, p));
            if (ok && c >= 2)
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(ypempty(c & 1), ((c >> 1) - 1) & 1, abort_flag, p));
            if (!ok) break;
#pragma unroll 2
            for (int tt = 0; tt < nt; ++tt) {
                const int t = c * C::TC + tt;
                // H_{t-1} W: the state as compensated hi + lo bf16 A fragments
                float acc[C::NT8][4];
    #pragma unroll
                for (int nt = 0; nt < C::NT8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    #pragma unroll
                for (int ks = 0; ks < C::KSTEPS; ++ks) {
                    uint32_t ahi[4], alo[4];
                    split_pack(h[2 * ks][0], h[2 * ks][1], ahi[0], alo[0]);
                    split_pack(h[2 * ks][2], h[2 * ks][3], ahi[1], alo[1]);
                    split_pack(h[2 * ks + 1][0], h[2 * ks + 1][1], ahi[2], alo[2]);
                    split_pack(h[2 * ks + 1][2], h[2 * ks + 1][3], ahi[3], alo[3]);
    #pragma unroll
                    for (int nt = 0; nt < C::NT8; ++nt) {
                        mma_bf16_16816(acc[nt], ahi, wb[ks][nt][0], wb[ks][nt][1]);
                        mma_bf16_16816(acc[nt], alo, wb[ks][nt][0], wb[ks][nt][1]);
                    }
                }
                // rank-1 term, tanh, gate blend
                const uint16_t* kt = reinterpret_cast<const uint16_t*>(st + C::ST_K + tt * K * 2);
                const uint16_t* qt = reinterpret_cast<const uint16_t*>(st + C::ST_Q + tt * K * 2);
                const uint32_t* vt = reinterpret_cast<const uint32_t*>(st + C::ST_V + tt * V * 2);
                const float gt = 1.f - *reinterpret_cast<const float*>(st + C::ST_F + tt * 4);
                const float k0 = bf16lo_to_f32(kt[i0]), k1 = bf16lo_to_f32(kt[i1]);
    #pragma unroll
                for (int nt = 0; nt < C::NT8; ++nt) {
                    const uint32_t vv = vt[4 * nt + tq];   // v[8nt + 2tq], v[8nt + 2tq + 1]
                    const float v0 = bf16lo_to_f32(vv), v1 = bf16hi_to_f32(vv);
                    const float a0 = fmaf(k0, v0, acc[nt][0]), a1 = fmaf(k0, v1, acc[nt][1]);
                    const float a2 = fmaf(k1, v0, acc[nt][2]), a3 = fmaf(k1, v1, acc[nt][3]);
                    // tanh accurate near zero in relative terms: this kernel also
                    // writes checkpoints for the backward
                    const float2 z01 = tanh2_acc(make_float2(a0, a1)), z23 = tanh2_acc(make_float2(a2, a3));
                    h[nt][0] = fmaf(gt, z01.x - h[nt][0], h[nt][0]);
                    h[nt][1] = fmaf(gt, z01.y - h[nt][1], h[nt][1]);
                    h[nt][2] = fmaf(gt, z23.x - h[nt][2], h[nt][2]);
                    h[nt][3] = fmaf(gt, z23.y - h[nt][3], h[nt][3]);
                }
                // readout partial over this warp's 16 rows: per column, q_i0 H[i0] + q_i1 H[i1],
                // then a reduce-scatter over the 8 lanes of a column group (lane bits 2-4)
                // that leaves lane (g, tq) with columns 8g + 2tq and 8g + 2tq + 1
                {
                    const float q0 = bf16lo_to_f32(qt[i0]), q1 = bf16lo_to_f32(qt[i1]);
                    float pr[2 * C::NT8];
    #pragma unroll
                    for (int nt = 0; nt < C::NT8; ++nt) {
                        pr[2 * nt] = fmaf(q1, h[nt][2], q0 * h[nt][0]);
                        pr[2 * nt + 1] = fmaf(q1, h[nt][3], q0 * h[nt][1]);
                    }
    #pragma unroll
                    for (int lvl = 0; lvl < 3; ++lvl) {
                        const int m = 16 >> lvl, n = 16 >> lvl;   // lane mask; live values 16, 8, 4
                        const bool up = (lane & m) != 0;
    #pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            if (i < n / 2) {
                                const float send = up ? pr[i] : pr[i + n / 2];
                                const float keep = up ? pr[i + n / 2] : pr[i];
                                pr[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                            }
                        }
                    }
                    float* yb = reinterpret_cast<float*>(smem + C::OFF_Y + (c & 1) * C::YBUF_BYTES);
                    *reinterpret_cast<float2*>(yb + (warp * C::TC + tt) * V + 8 * g + 2 * tq) = make_float2(pr[0], pr[1]);
                }
                if (t + 1 == ck_next) {   // checkpoint ck_idx = H_{t+1} (ck_next lies past T without checkpoints)
                    ck_next += p.C;
                    ++ck_idx;
                    if ((t + 1) < T) store_state(p.ckpt + ((size_t)bh * nck + ck_idx) * K * V);
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(in_empty(s));
                mbar_arrive(ypfull(c & 1));
            }
        }
        if (ok && p.HT != nullptr) store_state(p.HT + sbase);
    } else if (warp == C::W_PROD) {
        // ------------------------------------------------------------ producer
        const int qkb = qk_pair(p, bh);   // k / q rows of this pair's head group
        int last = -1;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % C::S;
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
                const uint32_t kb = (uint32_t)(nt * K * 2), vb = (uint32_t)(nt * V * 2);
                mbar_arrive_expect_tx(in_full(s), 2 * kb + vb);
                bulk_g2s(smem_u32(st + C::ST_K), static_cast<const uint16_t*>(p.k) + ((size_t)qkb * T + t0) * K, kb,
                         in_full(s));
                bulk_g2s(smem_u32(st + C::ST_Q), static_cast<const uint16_t*>(p.q) + ((size_t)qkb * T + t0) * K, kb,
                         in_full(s));
                bulk_g2s(smem_u32(st + C::ST_V), static_cast<const uint16_t*>(p.v) + ((size_t)bh * T + t0) * V, vb,
                         in_full(s));
            }
            last = c;
        }
        if (lane == 0)
            for (int c = max(0, last - C::S + 1); c <= last; ++c) mbar_wait_drain(in_full(c % C::S), (c / C::S) & 1, p);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ y storer
        for (int c = 0; c < nchunks; ++c) {
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(ypfull(c & 1), (c >> 1) & 1, abort_flag, p));
            if (!ok) break;
            const int t0 = c * C::TC, nt = min(C::TC, T - t0);
            const float* yb = reinterpret_cast<const float*>(smem + C::OFF_Y + (c & 1) * C::YBUF_BYTES);
            float* yg = p.y + ((size_t)bh * T + t0) * V;
            for (int e = lane * 4; e < nt * V; e += 128) {
                float4 a = *reinterpret_cast<const float4*>(yb + e);
#pragma unroll
                for (int w = 1; w < C::NW; ++w) {
                    const float4 b = *reinterpret_cast<const float4*>(yb + w * C::TC * V + e);
                    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
                }
                *reinterpret_cast<float4*>(yg + e) = a;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(ypempty(c & 1));
        }
    }
}

bool fwd_mma_supported(int K, int V) { return V == 64 && (K == 16 || K == 32 || K == 64); }

template <int K>
static cudaError_t launch_fwd_mma_k(const Params& p, cudaStream_t stream) {
    using C = FwdMmaCfg<K>;
    auto kern = m2rnn_fwd_mma_kernel<K>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<p.B * p.H, C::NTHREADS, C::SMEM_BYTES, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_fwd_mma(const Params& p, cudaStream_t s) {
    if (!fwd_mma_supported(p.K, p.V)) return cudaErrorNotSupported;
    switch (p.K) {
        case 16: return launch_fwd_mma_k<16>(p, s);
        case 32: return launch_fwd_mma_k<32>(p, s);
        case 64: return launch_fwd_mma_k<64>(p, s);
    }
    return cudaErrorNotSupported;
}

}  // namespace m2rnn
