// M²RNN forward scan on the sm_100a tensor cores (tcgen05).
//
// Recurrence (gist.science technical summary of "M²RNN: Non-Linear RNNs with
// Matrix-Valued States for Scalable Language Modeling", §2.1):
//   Z_t = tanh(H_{t-1} W + k_t v_tᵀ),  H_t = f_t H_{t-1} + (1 - f_t) Z_t,
// plus the readout y_t = H_tᵀ q_t (this library's reading; the pages define
// none).  The pages parallelise the forward over batch × head with each SM
// owning independent matrix states (§2.2); here one CTA owns one (b, h) pair
// for all T steps, with the fp32 state in registers.  When there are too few
// pairs to fill the GPU, a pair's K rows are split over several CTAs (the
// rows of H are independent given W, v_t and f_t) and the slices' partial
// readouts are summed by m2rnn_y_reduce_kernel; for 64-column states with at
// most 148 CTAs of 8 rows the row kernel of fwd_rows.cu takes the problem
// instead (launch_fwd_tc dispatches).
//
// Formulation.  The kernel computes the transpose of the transition GEMM,
//   D = Wᵀ · H_{t-1}ᵀ   (M = V columns of H, N = state rows, contraction V),
// so that tensor-memory lane j holds column j of H_{t-1}W.  Each epilogue
// thread therefore owns one column j of the state and a block of its rows:
// the rank-1 term k_t[i] v_t[j], the tanh, the gate blend and the readout
// y_t[j] = Σ_i q_t[i] H_t[i, j] are all thread-local (the readout needs one
// shuffle when a column is split over two half-warps).
//
//   A = Wᵀ      : shared memory, K-major, loaded once (bf16).
//   B = H_{t-1}ᵀ: shared memory, MN-major, rewritten each step by the
//                 epilogue.  The fp32 state is passed as a compensated pair
//                 hi + lo of bf16 operands (hi = the top 16 bits of the fp32
//                 word, lo = bf16(x - hi)), stacked along N, so one MMA
//                 produces both products and the epilogue adds them.
//   D           : tensor memory (fp32).
//
// Latency structure (measured on B200): a tcgen05.mma costs at least ~50-70
// cycles, and issue -> commit -> mbarrier wake-up adds ~400 cycles, so a
// step is bound by that round trip plus the epilogue, not by tensor
// throughput.  The state rows of a pair are therefore split into P = 2 tiles
// (4 at K = V = 128) whose chains run concurrently (ping-pong): while the
// epilogue warps of one tile run tanh and the blend, the tensor core computes
// another tile's product.  Two warps per TMEM lane quarter serve each tile (when the tile
// has enough rows), so that each thread handles few rows.
//
// Warp roles: warps [0, P·WPT) epilogue (warp w serves tile w / WPT, TMEM
// lane quarter w % 4 and row group (w % WPT) / 4), then one bulk-copy
// producer warp (k, q, v and f for TC steps per ring stage), one MMA warp
// (also owns the TMEM allocation) and one storer warp that sums the partial
// readouts and writes y.
//
// Input variants are resolved where the producer loads a step's inputs: with
// grouped k and q the pair reads the rows of its head group (qk_pair), and
// with gate logits the ring receives f_t = 1 / (1 + exp(-a_t)) (gate_value),
// so the epilogue is the same for every variant.  The epilogue's elementwise
// arithmetic runs on packed fp32 pairs (FADD2 / FFMA2), except in the
// fast-tanh kernel at V = 128, where the scalar loop measured faster.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace m2rnn {

// NSPLIT: bf16 terms of the state operand, 2 (hi + lo, ~2^-17 of each value)
// or 3 (hi + mid + lo, ~2^-26), the latter for the instantiation that writes
// the backward's checkpoints.
template <int K_, int V_, bool FAST_ = false, int NSPLIT_ = 2>
struct FwdTcCfg {
    static constexpr int K = K_, V = V_, NSPLIT = NSPLIT_;
    // row tiles with independent chains: 4 at K = V = 128 with the accurate
    // tanh, where the epilogue (32 rows per thread) and the MMA (N = 128 per
    // tile) are both long enough that two more chains in flight pay (8.86 ->
    // 7.70 ms at B = 4, 32 heads, T = 4096, bit-identical results); 2
    // elsewhere (the fast-tanh kernel at K = V = 128: 6.10 -> 7.34 ms with 4;
    // four 16-row tiles at K = V = 64 measured 17% slower)
    static constexpr int P = (V == 128 && K == 128 && !FAST_) ? 4 : 2;
    static constexpr int MPAD = V <= 64 ? 64 : 128;
    static constexpr int R = K / P;                       // state rows per tile
    static constexpr int NT = NSPLIT * R;                 // MMA N per tile (hi rows, [mid rows,] lo rows)
    // row groups per tile served by separate warps of the same lane quarter,
    // so that each thread handles at most 16 rows (measured on B200 at
    // K = V = 64: 1.85 -> 1.75 ms per 2048-step scan of 128 (b, h) pairs)
    static constexpr int SUBS = P == 4 ? 1 : (MPAD == 128 || K >= 64) ? 2 : 1;
    static constexpr int WPT = 4 * SUBS;                  // epilogue warps per tile
    static constexpr int RT = (MPAD == 64) ? R / (2 * SUBS) : R / SUBS;  // rows per thread
    // rows per tensor-memory load (8 with the three-term operand at 32 rows per
    // thread, which otherwise spills registers: 10.05 -> 9.85 ms for the 7B-MoE
    // training shape's forward)
    static constexpr int CH = (NSPLIT == 3 && RT > 8) ? 8 : RT < 16 ? RT : 16;
    // steps per ring stage (8 for the three-term operand at V = 128, for shared memory)
    static constexpr int TC = (NSPLIT == 3 && V == 128) ? 8 : 16;
    static constexpr int S = 4;                           // ring stages
    static constexpr int NWE = P * WPT;                   // epilogue warps
    static constexpr int W_PROD = NWE, W_MMA = NWE + 1, W_STORE = NWE + 2;
    static constexpr int NTHREADS = (NWE + 3) * 32;
    static constexpr int NSLOT = P * SUBS;                // readout partials per (t, j)

    static constexpr int A_BYTES = MPAD * V * 2;
    static constexpr int B_BYTES = NT * V * 2;
    static constexpr int ST_K = 0;
    static constexpr int ST_Q = TC * K * 2;
    static constexpr int ST_V = 2 * TC * K * 2;
    static constexpr int ST_F = ST_V + TC * V * 2;
    static constexpr int STAGE_BYTES = ((ST_F + TC * 4) + 127) / 128 * 128;
    static constexpr int YBUF_BYTES = NSLOT * TC * V * 4;

    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + A_BYTES;
    static constexpr int OFF_RING = OFF_B + P * B_BYTES;
    static constexpr int OFF_Y = OFF_RING + S * STAGE_BYTES;
    static constexpr int OFF_BAR = OFF_Y + 2 * YBUF_BYTES;
    static constexpr int NBAR = 2 * S + 2 * P + 4;
    static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16;
    static constexpr int TMEM_COLS = (P * NT <= 32) ? 32 : (P * NT <= 64) ? 64 : (P * NT <= 128) ? 128
                                   : (P * NT <= 256) ? 256 : 512;

    static_assert(K % (2 * P) == 0 && RT >= 4 && RT % 4 == 0, "unsupported K");
    static_assert(NTHREADS <= 1024, "block size");
    static_assert((MPAD == 64 && NT % 8 == 0) || (MPAD == 128 && NT % 16 == 0), "bad MMA N");
    static_assert(NT <= 256 && V % 16 == 0 && P * NT <= 512, "bad shape");
    static_assert(RT % CH == 0, "chunking");
    static_assert(SMEM_BYTES <= 227 * 1024, "smem");
};

// Operand terms of an instantiation: three when it writes checkpoints and the
// MMA shape allows N = 3R (M = 128 needs N % 16 == 0), else two.
template <int K, int V, bool FAST, bool CKPT>
__host__ __device__ constexpr int fwd_split() {
    using C2 = FwdTcCfg<K, V, FAST, 2>;
    return CKPT && (C2::MPAD == 64 || (3 * C2::R) % 16 == 0) ? 3 : 2;
}

// Three-term state operand: hi = RN(x), mid = RN(x - hi), lo = RN(x - hi - mid)
// in bf16 (each residual exact in fp32), at rows n, R + n and 2R + n of the
// layout of write_state_operand.
template <class C>
__device__ __forceinline__ void write_state_operand3(uint8_t* Bt, const float (&h)[C::RT], int j, int nloc) {
    auto split3 = [](float a, float b, uint32_t& hi, uint32_t& md, uint32_t& lo) {
        const __nv_bfloat162 hp = __floats2bfloat162_rn(a, b);
        hi = *reinterpret_cast<const uint32_t*>(&hp);
        const float a1 = a - bf16lo_to_f32(hi), b1 = b - bf16hi_to_f32(hi);
        const __nv_bfloat162 mp = __floats2bfloat162_rn(a1, b1);
        md = *reinterpret_cast<const uint32_t*>(&mp);
        const __nv_bfloat162 lp = __floats2bfloat162_rn(a1 - bf16lo_to_f32(md), b1 - bf16hi_to_f32(md));
        lo = *reinterpret_cast<const uint32_t*>(&lp);
    };
    uint8_t* colbase = Bt + (j >> 3) * (C::NT * 16) + (j & 7) * 16;
    if constexpr (C::RT % 8 == 0) {
#pragma unroll
        for (int g = 0; g < C::RT / 8; ++g) {
            uint4 hi, md, lo;
            split3(h[8 * g + 0], h[8 * g + 1], hi.x, md.x, lo.x);
            split3(h[8 * g + 2], h[8 * g + 3], hi.y, md.y, lo.y);
            split3(h[8 * g + 4], h[8 * g + 5], hi.z, md.z, lo.z);
            split3(h[8 * g + 6], h[8 * g + 7], hi.w, md.w, lo.w);
            const int n = nloc + 8 * g;
            *reinterpret_cast<uint4*>(colbase + (n >> 3) * 128) = hi;
            *reinterpret_cast<uint4*>(colbase + ((C::R + n) >> 3) * 128) = md;
            *reinterpret_cast<uint4*>(colbase + ((2 * C::R + n) >> 3) * 128) = lo;
        }
    } else {
        uint2 hi, md, lo;
        split3(h[0], h[1], hi.x, md.x, lo.x);
        split3(h[2], h[3], hi.y, md.y, lo.y);
        const int n = nloc;
        *reinterpret_cast<uint2*>(colbase + (n >> 3) * 128 + (n & 7) * 2) = hi;
        *reinterpret_cast<uint2*>(colbase + ((C::R + n) >> 3) * 128 + ((C::R + n) & 7) * 2) = md;
        *reinterpret_cast<uint2*>(colbase + ((2 * C::R + n) >> 3) * 128 + ((2 * C::R + n) & 7) * 2) = lo;
    }
}
template <class C>
__device__ __forceinline__ void write_operand(uint8_t* Bt, const float (&h)[C::RT], int j, int nloc) {
    if constexpr (C::NSPLIT == 3) write_state_operand3<C>(Bt, h, j, nloc);
    else write_state_operand<C>(Bt, h, j, nloc);
}

// FAST: tanh.approx.f32 (one SFU operation, ~2^-11 relative error) instead
// of the exp-based formula; forward-only inference mode.  CKPT: the
// instantiation launched when the call writes checkpoints; it finds the
// checkpoint steps by a running count (the general path's per-step remainder
// by the run-time stride cost ~200 cycles per step: 1.71 -> 1.58 ms on the
// 410M layer).  The other instantiation keeps the general path, whose
// run-time test never fires without checkpoints; dropping that code altogether
// measured slower at V = 128 (8.83 -> 9.15 ms) and equal at V = 64.
template <int K, int V, bool FAST, bool CKPT>
__global__ void __launch_bounds__(FwdTcCfg<K, V, FAST>::NTHREADS, 1) m2rnn_fwd_tc_kernel(const Params p) {
    using C = FwdTcCfg<K, V, FAST, fwd_split<K, V, FAST, CKPT>()>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // One CTA per (b, h) and slice of K rows (p.slices slices of the p.K state
    // rows: rows of H evolve independently given W, v_t and f_t).
    const int nsl = p.slices;
    const int bh = blockIdx.x / nsl, sl = blockIdx.x % nsl;
    const int KF = p.K, koff = sl * K;
    const int hd = bh % p.H;
    const int T = p.T;
    const int nchunks = (T + C::TC - 1) / C::TC;
    const int nck = (T + p.C - 1) / p.C;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    auto in_full = [&](int s) { return bar(s); };
    auto in_empty = [&](int s) { return bar(C::S + s); };
    auto bready = [&](int t) { return bar(2 * C::S + t); };
    auto accfull = [&](int t) { return bar(2 * C::S + C::P + t); };
    auto ypfull = [&](int i) { return bar(2 * C::S + 2 * C::P + i); };
    auto ypempty = [&](int i) { return bar(2 * C::S + 2 * C::P + 2 + i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::S; ++s) {
            mbar_init(in_full(s), 1);
            mbar_init(in_empty(s), C::NWE);
        }
        for (int t = 0; t < C::P; ++t) {
            mbar_init(bready(t), C::WPT);
            mbar_init(accfull(t), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(ypfull(i), C::NWE);
            mbar_init(ypempty(i), 1);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    // A = Wᵀ (K-major, no swizzle): element (m = j, k = l) = W[l][j] at
    // (j/8)·(V·16) + (l/8)·128 + (j%8)·16 + (l%8)·2; rows j >= V are zero.
    {
        const uint16_t* Wg = static_cast<const uint16_t*>(p.W) + (size_t)hd * V * V;
        for (int idx = threadIdx.x; idx < C::MPAD * V; idx += C::NTHREADS) {
            const int l = idx / C::MPAD, j = idx % C::MPAD;
            const uint16_t w = (j < V) ? Wg[l * V + j] : (uint16_t)0;
            *reinterpret_cast<uint16_t*>(smem + C::OFF_A + (j >> 3) * (V * 16) + (l >> 3) * 128 + (j & 7) * 16 +
                                         (l & 7) * 2) = w;
        }
    }
    fence_proxy_async_smem();
    if (warp == C::W_MMA) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < C::NWE) {
        // ------------------------------------------------------------ epilogue
        const int tile = warp / C::WPT, sub = (warp % C::WPT) >> 2, qd = warp & 3;
        const int half = (C::MPAD == 64) ? (lane >> 4) : 0;
        const int j = (C::MPAD == 64) ? qd * 16 + (lane & 15) : qd * 32 + lane;
        const bool jv = j < V;
        const int nsub = sub * (C::R / C::SUBS);  // first tile row of this warp
        const int nloc = nsub + half * C::RT;     // first tile row of this thread
        const int row0 = tile * C::R + nloc;      // first state row of this thread
        const int slot = tile * C::SUBS + sub;
        const size_t sbase = ((size_t)bh * KF + koff) * V;   // this slice's rows of H0 / H_T
        uint8_t* Bt = smem + C::OFF_B + tile * C::B_BYTES;

        float h[C::RT];
#pragma unroll
        for (int r = 0; r < C::RT; ++r) h[r] = (p.H0 != nullptr && jv) ? p.H0[sbase + (size_t)(row0 + r) * V + j] : 0.f;
        if ((CKPT || p.ckpt != nullptr) && jv) {
            float* ck = p.ckpt + (size_t)bh * nck * KF * V + (size_t)koff * V;
#pragma unroll
            for (int r = 0; r < C::RT; ++r) ck[(size_t)(row0 + r) * V + j] = h[r];
        }
        if (jv) write_operand<C>(Bt, h, j, nloc);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bready(tile));

        const uint32_t tbase = tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(tile * C::NT + nsub);
        int ck_next = p.C, ck_idx = 0;   // CKPT: the next checkpoint step and its index
        bool ok = true;
        // One step of the tile's chain: t is the step, tt its index in chunk c of
        // the ring, st the ring stage; false when the wait for the product
        // aborted.
        auto step = [&](int t, int tt, int c, const uint8_t* st) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(accfull(tile), t & 1, abort_flag, p))) return false;
            tc_fence_after();

            const float vj = jv ? bf16lo_to_f32(*reinterpret_cast<const uint16_t*>(st + C::ST_V + tt * V * 2 + j * 2))
                                : 0.f;
            const float g = 1.f - *reinterpret_cast<const float*>(st + C::ST_F + tt * 4);
            const uint16_t* kt = reinterpret_cast<const uint16_t*>(st + C::ST_K + tt * K * 2) + row0;
#pragma unroll
            for (int c0 = 0; c0 < C::RT; c0 += C::CH) {
                uint32_t ahi[C::CH], alo[C::CH], amd[C::CH];
                if constexpr (C::MPAD == 64) {
                    // the two half-warps own rows [0, RT) and [RT, 2RT) of the warp's block
                    tmem_ld_16x32bx2<C::CH, C::RT>(tbase + c0, ahi);
                    tmem_ld_16x32bx2<C::CH, C::RT>(tbase + (C::NSPLIT - 1) * C::R + c0, alo);
                    if constexpr (C::NSPLIT == 3) tmem_ld_16x32bx2<C::CH, C::RT>(tbase + C::R + c0, amd);
                } else {
                    tmem_ld_32x32b<C::CH>(tbase + c0, ahi);
                    tmem_ld_32x32b<C::CH>(tbase + (C::NSPLIT - 1) * C::R + c0, alo);
                    if constexpr (C::NSPLIT == 3) tmem_ld_32x32b<C::CH>(tbase + C::R + c0, amd);
                }
                float kk[C::CH];
                lds_bf16<C::CH>(kt + c0, kk);
                tc_wait_ld();
                reg_fence(ahi);
                reg_fence(alo);
                if constexpr (C::NSPLIT == 3) {
                    // the mid and lo products first, then the hi product
                    reg_fence(amd);
#pragma unroll
                    for (int r = 0; r < C::CH; ++r)
                        alo[r] = __float_as_uint(__uint_as_float(amd[r]) + __uint_as_float(alo[r]));
                }
                if constexpr (FAST && C::MPAD == 128) {
                    // scalar: with the single-SFU tanh at V = 128 the packed form
                    // below measured 6% slower (6.07 -> 6.43 ms at B = 4, 32 heads,
                    // K = V = 128, T = 4096); results are the same bits either way
#pragma unroll
                    for (int r = 0; r < C::CH; ++r) {
                        float a = __uint_as_float(ahi[r]) + __uint_as_float(alo[r]);
                        a = fmaf(kk[r], vj, a);
                        const float z = tanh_approx(a);
                        h[c0 + r] = fmaf(g, z - h[c0 + r], h[c0 + r]);
                    }
                } else {
                    // element pairs in packed fp32 instructions (the same rn operations
                    // as scalar code): 1.733 -> 1.713 ms at K = V = 64 and 9.25 -> 8.81 ms
                    // at K = V = 128 with the accurate tanh; the accurate tanh itself on
                    // pairs too (tanh2_ex2, the same bits as tanh_exp): 1.50 -> 1.43 ms
                    // and 7.68 -> 7.25 ms.  The instantiation that writes the
                    // backward's checkpoints takes tanh2_acc (the Taylor series below
                    // |x| = 1/8): the exp form's absolute error of ~2e-7 is a large
                    // relative error on small states, which heads whose recurrence
                    // amplifies perturbations carry into the gradients (the 7B-MoE
                    // shape's head 25: 4.1e-2 relative against 3.3e-3; 1.48 -> 1.52 ms
                    // at the 410M training workload)
                    const float2 vj2 = make_float2(vj, vj), g2 = make_float2(g, g);
#pragma unroll
                    for (int r = 0; r < C::CH; r += 2) {
                        float2 a2 = __fadd2_rn(make_float2(__uint_as_float(ahi[r]), __uint_as_float(ahi[r + 1])),
                                               make_float2(__uint_as_float(alo[r]), __uint_as_float(alo[r + 1])));
                        a2 = __ffma2_rn(make_float2(kk[r], kk[r + 1]), vj2, a2);
                        const float2 z2 = FAST   ? make_float2(tanh_approx(a2.x), tanh_approx(a2.y))
                                         : CKPT ? tanh2_acc(a2) : tanh2_ex2(a2);
                        const float2 d2 = __fadd2_rn(z2, make_float2(-h[c0 + r], -h[c0 + r + 1]));
                        const float2 h2 = __ffma2_rn(g2, d2, make_float2(h[c0 + r], h[c0 + r + 1]));
                        h[c0 + r] = h2.x;
                        h[c0 + r + 1] = h2.y;
                    }
                }
            }
            tc_fence_before();
            if (t + 1 < T) {
                if (jv) write_operand<C>(Bt, h, j, nloc);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bready(tile));
            }
            // readout partial over this thread's rows (off the critical path)
            {
                float qq[C::RT];
                lds_bf16<C::RT>(reinterpret_cast<const uint16_t*>(st + C::ST_Q + tt * K * 2) + row0, qq);
                float yp = 0.f;
#pragma unroll
                for (int r = 0; r < C::RT; ++r) yp = fmaf(qq[r], h[r], yp);
                if constexpr (C::MPAD == 64) yp += __shfl_xor_sync(0xffffffffu, yp, 16);
                if (half == 0 && jv)
                    reinterpret_cast<float*>(smem + C::OFF_Y + (c & 1) * C::YBUF_BYTES)[(slot * C::TC + tt) * V + j] = yp;
            }
            if constexpr (CKPT) {
                if (t + 1 == ck_next) {   // checkpoint ck_idx = H_{t+1}
                    ck_next += p.C;
                    ++ck_idx;
                    if (jv && (t + 1) < T) {
                        float* ck = p.ckpt + ((size_t)bh * nck + ck_idx) * KF * V + (size_t)koff * V;
#pragma unroll
                        for (int r = 0; r < C::RT; ++r) ck[(size_t)(row0 + r) * V + j] = h[r];
                    }
                }
            } else if (p.ckpt != nullptr && jv && (t + 1) < T && ((t + 1) % p.C) == 0) {
                float* ck = p.ckpt + ((size_t)bh * nck + (t + 1) / p.C) * KF * V + (size_t)koff * V;
#pragma unroll
                for (int r = 0; r < C::RT; ++r) ck[(size_t)(row0 + r) * V + j] = h[r];
            }
            return true;
        };
        auto wait_chunk = [&](int c, int s) {
            bool w = __all_sync(0xffffffffu, mbar_wait_bounded(in_full(s), (c / C::S) & 1, abort_flag, p));
            if (w && c >= 2)
                w = __all_sync(0xffffffffu, mbar_wait_bounded(ypempty(c & 1), ((c >> 1) - 1) & 1, abort_flag, p));
            return w;
        };
        auto release_chunk = [&](int c, int s) {
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(in_empty(s));
                mbar_arrive(ypfull(c & 1));
            }
        };
        if constexpr (CKPT && V == 64) {
            // the checkpointing forward of 64-column states: one chunk of steps
            // per outer iteration, the ring waits outside the step loop, which is
            // unrolled by 2 (1.58 -> 1.57 ms at the 410M training workload; the
            // same form measured slower without checkpoints, 1.50 -> 1.68 ms, and
            // at V = 128)
            for (int c = 0; c < nchunks && ok; ++c) {
                const int s = c % C::S, nt = min(C::TC, T - c * C::TC);
                const uint8_t* st = smem + C::OFF_RING + s * C::STAGE_BYTES;
                ok = wait_chunk(c, s);
                if (!ok) break;
#pragma unroll 2
                for (int tt = 0; tt < nt; ++tt) {
                    ok = step(c * C::TC + tt, tt, c, st);
                    if (!ok) break;
                }
                if (!ok) break;
                release_chunk(c, s);
            }
        } else {
            for (int t = 0; t < T; ++t) {
                const int c = t / C::TC, tt = t - c * C::TC, s = c % C::S;
                const uint8_t* st = smem + C::OFF_RING + s * C::STAGE_BYTES;
                if (tt == 0) {
                    ok = wait_chunk(c, s);
                    if (!ok) break;
                }
                ok = step(t, tt, c, st);
                if (!ok) break;
                if (tt == C::TC - 1 || t == T - 1) release_chunk(c, s);
            }
        }
        if (ok && p.HT != nullptr && jv) {
#pragma unroll
            for (int r = 0; r < C::RT; ++r) p.HT[sbase + (size_t)(row0 + r) * V + j] = h[r];
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
                const uint32_t kb = (uint32_t)(nt * K * 2), vb = (uint32_t)(nt * V * 2);
                mbar_arrive_expect_tx(in_full(s), 2 * kb + vb);
                if (nsl == 1) {
                    bulk_g2s(smem_u32(st + C::ST_K), static_cast<const uint16_t*>(p.k) + ((size_t)qkb * T + t0) * K, kb,
                             in_full(s));
                    bulk_g2s(smem_u32(st + C::ST_Q), static_cast<const uint16_t*>(p.q) + ((size_t)qkb * T + t0) * K, kb,
                             in_full(s));
                }
                bulk_g2s(smem_u32(st + C::ST_V), static_cast<const uint16_t*>(p.v) + ((size_t)bh * T + t0) * V, vb,
                         in_full(s));
            }
            if (nsl > 1) {
                // this slice's K values of each step's k and q row (strided in HBM)
                __syncwarp();
                if (lane < nt) {
                    const size_t r = ((size_t)qkb * T + t0 + lane) * KF + koff;
                    bulk_g2s(smem_u32(st + C::ST_K + lane * K * 2), static_cast<const uint16_t*>(p.k) + r, K * 2,
                             in_full(s));
                    bulk_g2s(smem_u32(st + C::ST_Q + lane * K * 2), static_cast<const uint16_t*>(p.q) + r, K * 2,
                             in_full(s));
                }
            }
            last = c;
        }
        // copies still in flight must land before the CTA exits
        if (lane == 0)
            for (int c = max(0, last - C::S + 1); c <= last; ++c) mbar_wait_drain(in_full(c % C::S), (c / C::S) & 1, p);
        __syncwarp();
    } else if (warp == C::W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(C::MPAD, C::NT, 0, 1);
            const uint32_t a0 = smem_u32(smem + C::OFF_A);
            int issued[C::P];
#pragma unroll
            for (int i = 0; i < C::P; ++i) issued[i] = -1;
            bool ok = true;
            for (int t = 0; t < T && ok; ++t) {
#pragma unroll
                for (int tile = 0; tile < C::P; ++tile) {
                    if (!mbar_wait_bounded(bready(tile), t & 1, abort_flag, p)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b0 = smem_u32(smem + C::OFF_B + tile * C::B_BYTES);
#pragma unroll
                    for (int ks = 0; ks < V / 16; ++ks) {
                        const uint64_t ad = smem_desc(a0 + ks * 256, 128, V * 16);
                        const uint64_t bd = smem_desc(b0 + ks * 2 * C::NT * 16, C::NT * 16, 128);
                        tc_mma_f16_ss(tmem + tile * C::NT, ad, bd, idesc, ks > 0 ? 1u : 0u);
                    }
                    tc_commit(accfull(tile));
                    issued[tile] = t;
                }
            }
#pragma unroll
            for (int tile = 0; tile < C::P; ++tile)
                if (issued[tile] >= 0) mbar_wait_drain(accfull(tile), issued[tile] & 1, p);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ y storer
        for (int c = 0; c < nchunks; ++c) {
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(ypfull(c & 1), (c >> 1) & 1, abort_flag, p));
            if (!ok) break;
            const int t0 = c * C::TC, nt = min(C::TC, T - t0);
            const float* yb = reinterpret_cast<const float*>(smem + C::OFF_Y + (c & 1) * C::YBUF_BYTES);
            // with several slices, each writes its partial readout; a fixed-order
            // sum over the slices follows (m2rnn_y_reduce_kernel)
            float* yout = nsl == 1 ? p.y : p.ypart + (size_t)sl * p.B * p.H * T * V;
            float* yg = yout + ((size_t)bh * T + t0) * V;
            for (int e = lane * 4; e < nt * V; e += 128) {
                float4 a = *reinterpret_cast<const float4*>(yb + e);
#pragma unroll
                for (int sl = 1; sl < C::NSLOT; ++sl) {
                    const float4 b = *reinterpret_cast<const float4*>(yb + sl * C::TC * V + e);
                    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
                }
                *reinterpret_cast<float4*>(yg + e) = a;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(ypempty(c & 1));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int K, int V, bool FAST, bool CKPT>
static cudaError_t launch_fwd_tc_one(const Params& p, cudaStream_t stream) {
    using C = FwdTcCfg<K, V, FAST, fwd_split<K, V, FAST, CKPT>()>;
    auto kern = m2rnn_fwd_tc_kernel<K, V, FAST, CKPT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<p.B * p.H * p.slices, C::NTHREADS, C::SMEM_BYTES, stream>>>(p);
    return cudaGetLastError();
}

template <int K, int V>
static cudaError_t launch_fwd_tc_kv(const Params& p, cudaStream_t stream) {
    if (p.ckpt != nullptr)
        return p.fast_tanh ? launch_fwd_tc_one<K, V, true, true>(p, stream)
                           : launch_fwd_tc_one<K, V, false, true>(p, stream);
    return p.fast_tanh ? launch_fwd_tc_one<K, V, true, false>(p, stream)
                       : launch_fwd_tc_one<K, V, false, false>(p, stream);
}

template <int K>
static cudaError_t launch_fwd_tc_k(const Params& p, cudaStream_t s) {
    switch (p.V) {
        case 16: return launch_fwd_tc_kv<K, 16>(p, s);
        case 32: return launch_fwd_tc_kv<K, 32>(p, s);
        case 64: return launch_fwd_tc_kv<K, 64>(p, s);
        case 128: return launch_fwd_tc_kv<K, 128>(p, s);
    }
    return cudaErrorInvalidValue;
}

// y = the sum of the slices' partial readouts, in slice order.
__global__ void m2rnn_y_reduce_kernel(const Params p) {
    const size_t n4 = (size_t)p.B * p.H * p.T * p.V / 4;
    const float4* part = reinterpret_cast<const float4*>(p.ypart);
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n4; e += (size_t)gridDim.x * blockDim.x) {
        float4 a = part[e];
        for (int sl = 1; sl < p.slices; ++sl) {
            const float4 b = part[sl * n4 + e];
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        reinterpret_cast<float4*>(p.y)[e] = a;
    }
}

int fwd_tc_slices(int B, int H, int K, int V) {
    // Few pairs of 64-column states: the row kernel (fwd_rows.cu), 8 rows per CTA.
    const int rs = fwd_rows_per_cta(B, H, K, V);
    if (rs > 0) return K / rs;
    // Otherwise rows are split only while the (b, h) pairs alone would leave
    // most SMs idle: a 16-row slice's step is ~1.45x shorter than a 64-row
    // CTA's (measured on B200 at V = 64: ~1000 vs ~1430 cycles per step).
    const long long pairs = (long long)B * H;
    int s = 1;
    while (s < 8 && K / (2 * s) >= 16 && pairs * 2 * s <= kNumSMs) s *= 2;
    return s;
}

cudaError_t launch_y_reduce(const Params& p, cudaStream_t s) {
    const size_t n4 = (size_t)p.B * p.H * p.T * p.V / 4;
    const int blocks = (int)((n4 + 255) / 256 < 1184 ? (n4 + 255) / 256 : 1184);
    m2rnn_y_reduce_kernel<<<blocks, 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_fwd_tc(const Params& p0, cudaStream_t s) {
    if (fwd_rows_per_cta(p0.B, p0.H, p0.K, p0.V) > 0) return launch_fwd_rows(p0, s);
    Params p = p0;
    p.slices = fwd_tc_slices(p.B, p.H, p.K, p.V);
    if (p.slices > 1) {
        cudaError_t e;
        switch (p.K / p.slices) {
            case 16: e = launch_fwd_tc_k<16>(p, s); break;
            case 32: e = launch_fwd_tc_k<32>(p, s); break;
            case 64: e = launch_fwd_tc_k<64>(p, s); break;
            default: return cudaErrorInvalidValue;
        }
        if (e != cudaSuccess) return e;
        return launch_y_reduce(p, s);
    }
    switch (p.K) {
        case 16: return launch_fwd_tc_k<16>(p, s);
        case 32: return launch_fwd_tc_k<32>(p, s);
        case 64: return launch_fwd_tc_k<64>(p, s);
        case 128: return launch_fwd_tc_k<128>(p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace m2rnn
