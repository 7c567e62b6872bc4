// M²RNN backward (BPTT) on the sm_100a tensor cores for every state shape and
// checkpoint stride the V = 64 kernel of bwd_tc.cu does not take: V in
// {16, 32, 128}, K = 16 at any V, and strides beyond that kernel's on-chip
// chunk.
//
// The chain rule of the recurrence (gist.science technical summary of
// "M²RNN: Non-Linear RNNs with Matrix-Valued States for Scalable Language
// Modeling", §2.1: Z_t = tanh(H_{t-1}W + k_t v_tᵀ), H_t = f_t H_{t-1} +
// (1-f_t) Z_t) and of the readout y_t = H_tᵀ q_t, with G_t = dL/dH_t:
//   G_t  += q_t dy_tᵀ            dq_t = H_t dy_t
//   dA_t  = (1 - f_t) G_t ⊙ (1 - Z_t²)
//   df_t  = <G_t, H_{t-1} - Z_t>  dk_t = dA_t v_t      dv_t = dA_tᵀ k_t
//   dW   += H_{t-1}ᵀ dA_t         G_{t-1} = f_t G_t + dA_t Wᵀ,   dH0 = G_0.
// As in bwd_tc.cu, each checkpoint chunk of C steps is recomputed from
// H_{c·C} with the forward's epilogue and the state as one bf16 operand (the
// pages' backward recomputes states rather than storing them, §2.2; the
// exact fp32 checkpoint every C <= 16 steps bounds that rounding), its states
// and Z's stay on chip for V = 128 (in tensor memory and a ring of bf16
// state operands, as in bwd_tc.cu: 32.7 -> 27.6 ms at the 7B-MoE training
// shape with C = 8) or go to a workspace scratch for the other shapes, and
// the chunk is then walked in reverse; the recompute of one
// chunk and the reverse walk of the next run interleaved, each chain with its
// own accumulators and MMA issuer.  Per step and tile three tcgen05 GEMMs:
//   recompute      D = Wᵀ · H_{t-1}ᵀ   (M = MX state columns, N = the tile's rows, bf16 state)
//   G-propagation  D = W · dA_tᵀ       (N = the tile's rows of dA, hi and lo)
//   dW             D_W += H_{t-1}ᵀ · dA_t  (M = MX, N = V), accumulated over the sequence
// with MX = 64 for V <= 64 (rows j >= V of the operands are zero) and 128 for
// V = 128.  What differs from the V = 64 kernel:
//  * One shared-memory copy of W serves both products.  With MX-row padding,
//    the K-major layout of Wᵀ and the MN-major layout of W put every element
//    W[l][j] at the same byte, (j/8)·MX·16 + (l/8)·128 + (j%8)·16 + (l%8)·2;
//    only the two descriptors differ.
//  * dk_t and dq_t are column sums (Σ_j dA[i,j] v[j], Σ_j H_t[i,j] dy[j]), and
//    M = MX leaves no spare operand row to put them on the tensor core, so
//    each thread forms its rows' products and a lane reduce-scatter over the
//    lanes that share those rows yields one row sum per lane group; the
//    storer warp adds the four lane quarters' partials in a fixed order.
//    dq_t is taken in the recompute step that produces H_t.
//  * V = 128 uses slices of at most 32 state rows (a thread then owns 8 rows
//    of one column; 16 would exceed the register file at this block size),
//    so a pair can span four CTAs; their dv and df partials go to the
//    workspace and m2rnn_slice_sum_kernel adds them in slice order.
// All sums run in fixed orders, so results are deterministic.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace m2rnn {

// OC: the recomputed chunk stays on chip (the Z's in tensor memory, the
// states in a ring of bf16 operands, as in bwd_tc.cu); for V = 128 with a
// checkpoint stride the tensor memory holds.  Otherwise the chunk goes
// through a global-memory scratch.
template <int KS_, int V_, bool OC_ = false>
struct BwdTcgCfg {
    static constexpr int K = KS_;             // state rows of this CTA's slice
    static constexpr int V = V_;
    static constexpr bool OC = OC_;
    static constexpr int MX = V <= 64 ? 64 : 128;   // M of every MMA; state columns j < V are real
    static constexpr int P = K >= 32 ? 2 : 1;       // row tiles with independent chains
    static constexpr int R = K / P;                 // rows per tile
    static constexpr int NT = 2 * R;                // MMA N per tile (hi rows, then lo rows)
    static constexpr int RT = 8;                    // rows per epilogue thread
    // M = 64: a lane quarter holds 16 columns and its two half-warps split the
    // rows; M = 128: 32 columns per quarter, one row block per warp
    static constexpr int SUBS = MX == 64 ? R / (2 * RT) : R / RT;
    static constexpr int WPT = 4 * SUBS;            // epilogue warps per tile
    static constexpr int NWE = P * WPT;             // epilogue warps
    static constexpr int NSLOT = P * SUBS;          // dv partials per (t, j)
    static constexpr int LG = MX == 64 ? 16 : 32;   // lanes that share a row block (one column each)
    // on chip: per step one TMEM column per thread and row, NSLOT·RT columns a
    // lane quarter, in the upper 256 columns
    static constexpr int SCR_COL = 256, SCR_STEP = NSLOT * RT;
    static constexpr int CMAX = OC ? (256 / SCR_STEP < 16 ? 256 / SCR_STEP : 16) : 16;   // max steps per chunk
    static constexpr int W_MREV = NWE, W_MREC = NWE + 1, W_STORE = NWE + 2, W_PROD = NWE + 3;
    static constexpr int NTHREADS = (NWE + 4) * 32;
    static constexpr int NSTAGE = 3;                // input chunks: recompute of i, reverse of i-1, prefetch of i+1

    static constexpr int W_BYTES = MX * MX * 2;     // W, zero-padded to MX x MX
    static constexpr int B_BYTES = NT * V * 2;      // one state / dA operand (hi and lo)
    static constexpr int BS_BYTES = MX * R * 2;     // H_{t-1} hi operand of the dW MMA (MX rows)
    static constexpr int NBR = CMAX + 2;            // on chip: state-operand ring slots (R rows each)
    static constexpr int ST_K = 0;                  // the slice's K values of k and q per step
    static constexpr int ST_Q = CMAX * K * 2;
    static constexpr int ST_V = 2 * CMAX * K * 2;
    static constexpr int ST_DY = ST_V + CMAX * V * 2;            // CMAX + 1 rows: row r is step c0 - 1 + r
    static constexpr int ST_F = ST_DY + (CMAX + 1) * V * 2;
    static constexpr int STAGE_BYTES = ((ST_F + CMAX * 4) + 127) / 128 * 128;
    static constexpr int DVP = 0;                                // [CMAX][NSLOT][V]
    static constexpr int DFP = DVP + CMAX * NSLOT * V * 4;       // [CMAX][NWE]
    static constexpr int DKP = DFP + CMAX * NWE * 4;             // [CMAX][4 quarters][K]
    static constexpr int PART_BYTES = DKP + CMAX * 4 * K * 4;
    static constexpr int DQ_BYTES = CMAX * 4 * K * 4;            // [CMAX][4 quarters][K]

    static constexpr int OFF_W = 0;
    static constexpr int OFF_BD = OFF_W + W_BYTES;               // dA operands per tile
    // recompute state operands per tile, then H_{t-1} hi operands per tile; on
    // chip instead one ring [NBR][P] of BS_BYTES operands serving both
    static constexpr int OFF_BR = OFF_BD + P * B_BYTES;
    static constexpr int OFF_BS = OFF_BR + (OC ? 0 : P * B_BYTES);
    static constexpr int BR_END = OC ? OFF_BR + NBR * P * BS_BYTES : OFF_BS + P * BS_BYTES;
    static constexpr int OFF_RING = (BR_END + 1023) / 1024 * 1024;
    static constexpr int OFF_CK = OFF_RING + NSTAGE * STAGE_BYTES;   // the next checkpoint (fp32 [K][V])
    static constexpr int OFF_PART = OFF_CK + K * V * 4;
    static constexpr int FIXED = OFF_PART + 512;                 // + barriers and the TMEM slot
    // dv / df / dk partials double-buffered (the storer's pass over one chunk
    // overlaps the next chunk's reverse walk) when shared memory allows; the
    // dq partials of a chunk are written one phase earlier, so they need one
    // buffer more than the others
    static constexpr int NPART = (FIXED + 2 * PART_BYTES + 3 * DQ_BYTES <= 227 * 1024) ? 2 : 1;
    static constexpr int NDQ = NPART + 1;
    static constexpr int OFF_DQ = OFF_PART + NPART * PART_BYTES;
    static constexpr int OFF_BAR = OFF_DQ + NDQ * DQ_BYTES;
    // in_full[3], in_empty[3], bready/accfull of both chains per tile,
    // pfull/pempty per partial buffer, ck_full/ck_empty
    static constexpr int NBAR = 2 * NSTAGE + 4 * P + 2 * NPART + 2;
    static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16;
    static constexpr int REV_COL = 0;                            // G-propagation accumulators, NT columns per tile
    static constexpr int REC_COL = P * NT;                       // recompute accumulators
    static constexpr int DW_COL = 2 * P * NT;                    // dW accumulator (V columns)
    static constexpr int TMEM_COLS = OC ? 512 : (DW_COL + V <= 64) ? 64 : (DW_COL + V <= 128) ? 128
                                   : (DW_COL + V <= 256) ? 256 : 512;

    static_assert(K == 16 || K == 32 || (K == 64 && MX == 64), "slice rows");
    static_assert(R == 16 || R == 32, "tile rows: the dW MMA takes 16-row k-steps");
    static_assert(SUBS >= 1 && NWE * 32 * RT == K * MX, "row split");
    static_assert((MX == 64 && NT % 8 == 0) || (MX == 128 && NT % 16 == 0), "N of the state MMAs");
    static_assert((MX == 64 && V % 8 == 0) || (MX == 128 && V % 16 == 0), "N of the dW MMA");
    static_assert(NTHREADS <= 1024, "block size");
    static_assert(DW_COL + V <= TMEM_COLS && TMEM_COLS <= 512, "TMEM columns");
    static_assert(!OC || (MX == 128 && DW_COL + V <= SCR_COL && CMAX * SCR_STEP <= 256 && CMAX >= 8),
                  "on-chip chunk: 128-column states, scratch above the accumulators");
    static_assert(OFF_W % 1024 == 0 && OFF_BR % 128 == 0 && OFF_BD % 128 == 0 && OFF_BS % 128 == 0 &&
                  OFF_RING % 128 == 0 && OFF_CK % 128 == 0 && OFF_PART % 16 == 0 && OFF_DQ % 16 == 0 &&
                  OFF_BAR % 8 == 0, "alignment of shared-memory regions");
    static_assert(SMEM_BYTES <= 227 * 1024, "smem");
};

// Writes the hi parts (bf16, round to nearest) of this thread's RT values of
// state column j, rows nloc .. nloc+RT-1, into the K-major A operand of the dW
// MMA: element (m = j, k = row n) at (j/8)·(R·16) + (n/8)·128 + (j%8)·16 + (n%8)·2.
template <class C>
__device__ __forceinline__ void write_dw_a_operand(uint8_t* Bs, const float (&h)[C::RT], int j, int nloc) {
    uint8_t* colbase = Bs + (j >> 3) * (C::R * 16) + (j & 7) * 16;
    auto pack = [](float a, float b) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<const uint32_t*>(&v);
    };
#pragma unroll
    for (int g = 0; g < C::RT / 8; ++g) {
        const uint4 hi = make_uint4(pack(h[8 * g], h[8 * g + 1]), pack(h[8 * g + 2], h[8 * g + 3]),
                                    pack(h[8 * g + 4], h[8 * g + 5]), pack(h[8 * g + 6], h[8 * g + 7]));
        *reinterpret_cast<uint4*>(colbase + ((nloc + 8 * g) >> 3) * 128) = hi;
    }
}

// Accumulator rows of this thread: the hi half of its RT rows.
template <class C>
__device__ __forceinline__ void load_acc_hi(uint32_t taddr, uint32_t (&hi)[C::RT]) {
    if constexpr (C::MX == 64) tmem_ld_16x32bx2<C::RT, C::RT>(taddr, hi);
    else tmem_ld_32x32b<C::RT>(taddr, hi);
}

// Accumulator rows of this thread (hi and lo halves of its RT rows).
template <class C>
__device__ __forceinline__ void load_acc(uint32_t taddr, uint32_t (&hi)[C::RT], uint32_t (&lo)[C::RT]) {
    if constexpr (C::MX == 64) {
        tmem_ld_16x32bx2<C::RT, C::RT>(taddr, hi);
        tmem_ld_16x32bx2<C::RT, C::RT>(taddr + C::R, lo);
    } else {
        tmem_ld_32x32b<C::RT>(taddr, hi);
        tmem_ld_32x32b<C::RT>(taddr + C::R, lo);
    }
}

// Sum over the lanes of a lane group (lanes that differ only in the bits of
// M, M/2, ..., 1) of the N values a[0..N) of each lane: a reduce-scatter that
// halves the values at each mask (a lane with the mask bit set keeps the upper
// half) until one is left, then a full reduction over the remaining masks.
// Returns the group sum of value `row`, which the lane learns; every lane of
// an aligned block of 2M/N lanes holds the same row.  Fixed order throughout.
template <int N, int M>
__device__ __forceinline__ float reduce_scatter(float* a, int lane, int& row) {
    if constexpr (N == 1) {
        float x = a[0];
#pragma unroll
        for (int m = M; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
        return x;
    } else {
        const bool up = (lane & M) != 0;
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            const float keep = up ? a[i + N / 2] : a[i];
            const float send = up ? a[i] : a[i + N / 2];
            a[i] = keep + __shfl_xor_sync(0xffffffffu, send, M);
        }
        if (up) row += N / 2;
        return reduce_scatter<N / 2, M / 2>(a, lane, row);
    }
}

template <int KS, int V, bool OC>
__global__ void __launch_bounds__(BwdTcgCfg<KS, V, OC>::NTHREADS, 1) m2rnn_bwd_tcg_kernel(const Params p) {
    using C = BwdTcgCfg<KS, V, OC>;
    constexpr int K = C::K;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nsl = p.slices;
    const int bh = blockIdx.x / nsl, sl = blockIdx.x % nsl;
    const int KF = K * nsl, koff = sl * K;   // all state rows of the pair; first row of this slice
    const int hd = bh % p.H;
    const int T = p.T, CS = p.C;
    const int nck = (T + CS - 1) / CS;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    auto in_full = [&](int s) { return bar(s); };
    auto in_empty = [&](int s) { return bar(C::NSTAGE + s); };
    auto bready_rev = [&](int t) { return bar(2 * C::NSTAGE + t); };
    auto accfull_rev = [&](int t) { return bar(2 * C::NSTAGE + C::P + t); };
    auto bready_rec = [&](int t) { return bar(2 * C::NSTAGE + 2 * C::P + t); };
    auto accfull_rec = [&](int t) { return bar(2 * C::NSTAGE + 3 * C::P + t); };
    auto pfull = [&](int b) { return bar(2 * C::NSTAGE + 4 * C::P + b); };
    auto pempty = [&](int b) { return bar(2 * C::NSTAGE + 4 * C::P + C::NPART + b); };
    const uint32_t ck_full = bar(2 * C::NSTAGE + 4 * C::P + 2 * C::NPART);
    const uint32_t ck_empty = bar(2 * C::NSTAGE + 4 * C::P + 2 * C::NPART + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(in_full(s), 1);
            mbar_init(in_empty(s), C::NWE);
        }
        for (int t = 0; t < C::P; ++t) {
            mbar_init(bready_rev(t), C::WPT);
            mbar_init(accfull_rev(t), 1);
            mbar_init(bready_rec(t), C::WPT);
            mbar_init(accfull_rec(t), 1);
        }
        for (int b = 0; b < C::NPART; ++b) {
            mbar_init(pfull(b), C::NWE);
            mbar_init(pempty(b), 1);
        }
        mbar_init(ck_full, 1);
        mbar_init(ck_empty, C::NWE);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    // Operands: zero everything (the padding rows of W and of the dW A operand
    // stay zero), then W[l][j] at (j/8)·MX·16 + (l/8)·128 + (j%8)·16 + (l%8)·2.
    for (int i = threadIdx.x; i < C::OFF_RING / 16; i += C::NTHREADS)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    {
        const uint16_t* Wg = static_cast<const uint16_t*>(p.W) + (size_t)hd * V * V;
        for (int idx = threadIdx.x; idx < V * V; idx += C::NTHREADS) {
            const int l = idx / V, j = idx % V;
            *reinterpret_cast<uint16_t*>(smem + C::OFF_W + (j >> 3) * (C::MX * 16) + (l >> 3) * 128 + (j & 7) * 16 +
                                         (l & 7) * 2) = Wg[l * V + j];
        }
    }
    fence_proxy_async_smem();
    if (warp == C::W_PROD) {
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
        const int half = C::MX == 64 ? (lane >> 4) : 0;
        const int j = C::MX == 64 ? qd * 16 + (lane & 15) : qd * 32 + lane;
        const bool jv = j < V;                      // a real state column (the rest carry zeros)
        const int nsub = sub * (C::R / C::SUBS);    // first tile row of this warp
        const int nloc = nsub + half * C::RT;       // first tile row of this thread
        const int row0 = tile * C::R + nloc;        // first slice row of this thread
        const int slot = tile * C::SUBS + sub;
        const size_t sbase = ((size_t)bh * KF + koff) * V;   // this slice's rows of dH_T / dH0
        uint8_t* Br = smem + C::OFF_BR + tile * C::B_BYTES;     // (not on chip)
        uint8_t* Bd = smem + C::OFF_BD + tile * C::B_BYTES;
        uint8_t* Bs = smem + C::OFF_BS + tile * C::BS_BYTES;    // (not on chip)
        // On chip: the Z's of the chunk in TMEM (thread l of warp w in lane
        // 32·(w mod 4) + l, columns SCR_COL + x·SCR_STEP + slot·RT + r for
        // scratch slot x), the states H_{c0+u} in a ring of bf16 operands of
        // R rows (this thread's values at brt, slot x at x·RING_STEP), which
        // the recompute MMA of step c0+u and the dW MMA of the same step read,
        // in the slot orders of bwd_tc.cu (scratch: u for even phases, CS-1-u
        // for odd ones; ring: u and CS+1-u).
        constexpr int RING_STEP = C::P * C::BS_BYTES;
        const int tpos = (j >> 3) * (C::R * 16) + (j & 7) * 16 + (nloc >> 3) * 128 + (nloc & 7) * 2;
        uint8_t* const brt = smem + C::OFF_BR + tile * C::BS_BYTES + tpos;
        const uint32_t scr = tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(C::SCR_COL + slot * C::RT);
        const uint32_t lanes = (uint32_t)(qd * 32) << 16;
        const uint32_t tb_rev = tmem + lanes + (uint32_t)(C::REV_COL + tile * C::NT + nsub);
        const uint32_t tb_rec = tmem + lanes + (uint32_t)(C::REC_COL + tile * C::NT + nsub);
        // Global scratch per CTA (not on chip): C slots of states H_{c0+u} and
        // C slots of Z_{c0+u}; the chunk recomputed in phase i stores step u in
        // slot u for even i and C-1-u for odd i, so the next phase's recompute
        // overwrites only slots the reverse walk has read.  Slot x of CTA b is
        // the block x·nCTA + b of K·MX values; thread t holds its RT values at
        // t·RT, and only the thread that wrote a value reads it back.
        const size_t nct = gridDim.x;
        const size_t blk = (size_t)K * C::MX;
        float* const Sst = p.scratch + (size_t)blockIdx.x * blk;
        float* const Sz = Sst + (size_t)CS * nct * blk;
        auto sslot = [&](int i, int u) { return (i & 1) ? CS - 1 - u : u; };
        const size_t tslot = (size_t)threadIdx.x * C::RT;
        const uint64_t pol_keep = l2_policy_evict_last();
        const bool v8 = (reinterpret_cast<uintptr_t>(Sst) & 31) == 0;
        auto st_vec = [&](float* base, int u, const float (&v)[C::RT]) {
            float* d = base + (size_t)u * nct * blk + tslot;
            if (v8) {
#pragma unroll
                for (int g = 0; g < C::RT / 8; ++g) st_global_v8_hint(d + 8 * g, v + 8 * g, pol_keep);
            } else {
#pragma unroll
                for (int g = 0; g < C::RT / 4; ++g)
                    st_global_v4_hint(d + 4 * g, v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3], pol_keep);
            }
        };
        auto ld_vec = [&](const float* base, int u, float (&v)[C::RT]) {
            const float* src = base + (size_t)u * nct * blk + tslot;
            if (v8) {
#pragma unroll
                for (int g = 0; g < C::RT / 8; ++g) ld_global_v8(src + 8 * g, v + 8 * g);
            } else {
                const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
                for (int g = 0; g < C::RT / 4; ++g) {
                    const float4 x = s4[g];
                    v[4 * g] = x.x; v[4 * g + 1] = x.y; v[4 * g + 2] = x.z; v[4 * g + 3] = x.w;
                }
            }
        };
        auto stage = [&](int i) { return smem + C::OFF_RING + (i % C::NSTAGE) * C::STAGE_BYTES; };
        auto bf16_at = [&](const uint8_t* st, int off) {
            return jv ? bf16lo_to_f32(*reinterpret_cast<const uint16_t*>(st + off + j * 2)) : 0.f;
        };
        // one row sum per lane group; lanes whose low bits are zero store it
        constexpr int WMASK = C::LG / 8 - 1;   // bits below the last reduce-scatter mask
        auto row_sum_store = [&](float (&pr)[C::RT], float* dst) {
            int rr = 0;
            const float s = reduce_scatter<C::RT, C::LG / 2>(pr, lane, rr);
            if ((lane & WMASK) == 0) dst[qd * K + tile * C::R + nloc + rr] = s;
        };

        float G[C::RT], h[C::RT], zc[C::RT], hpc[C::RT];
        uint32_t szr[C::RT];   // on chip: the Z's of the next reverse step as loaded from TMEM
#pragma unroll
        for (int r = 0; r < C::RT; ++r)
            G[r] = (p.dHT != nullptr && jv) ? p.dHT[sbase + (size_t)(row0 + r) * V + j] : 0.f;
        float fprev = 0.f;
        uint32_t nrev = 0, nrec = 0;   // accumulator-full events consumed per chain
        bool ok = true;
        for (int m = 0; m <= nck && ok; ++m) {
            // recompute: chunk m of the processing order (reverse time)
            const bool has_rec = m < nck;
            const int c0r = (nck - 1 - m) * CS;
            const int lenr = has_rec ? min(CS, T - c0r) : 0;
            const uint8_t* str = stage(m);
            float* const dqp = reinterpret_cast<float*>(smem + C::OFF_DQ + (m % C::NDQ) * C::DQ_BYTES);
            // reverse: chunk m-1
            const bool has_rev = m >= 1;
            const int c0v = (nck - m) * CS;
            const int lenv = has_rev ? min(CS, T - c0v) : 0;
            const uint8_t* stv = stage(m + C::NSTAGE - 1);
            const int pb = (m + C::NPART - 1) % C::NPART;   // partial-sum buffer of chunk m-1
            float* const part = reinterpret_cast<float*>(smem + C::OFF_PART + pb * C::PART_BYTES);
            // on chip: slot walks of this phase's recompute and reverse chunks
            const bool odd = (m & 1) != 0;
            uint8_t* const rec_ring = brt + (odd ? (CS + 1) * RING_STEP : 0);
            uint8_t* const rev_ring = brt + (odd ? 0 : (CS + 1) * RING_STEP);
            const int rec_rstep = odd ? -RING_STEP : RING_STEP;
            const uint32_t rec_scr = scr + (uint32_t)(odd ? (CS - 1) * C::SCR_STEP : 0);
            const uint32_t rev_scr = scr + (uint32_t)(odd ? 0 : (CS - 1) * C::SCR_STEP);
            const int rec_sstep = odd ? -C::SCR_STEP : C::SCR_STEP;
            auto load_rev = [&](int u) {   // the reverse step of chunk step u: its Z's and H_{t-1}
                if constexpr (C::OC) {
                    tc_wait_st();
                    tmem_ld_32x32b<C::RT>(rev_scr - (uint32_t)(u * rec_sstep), szr);
                    get_state_hi<C>(rev_ring - u * rec_rstep, hpc);
                } else {
                    ld_vec(Sz, sslot(m - 1, u), zc);
                    ld_vec(Sst, sslot(m - 1, u), hpc);
                }
            };

            if (has_rev) {
                const int i = m - 1;
                // the storer is done with chunk i - NPART (its dv / df / dk buffer,
                // and the dq buffer of chunk i - NPART = m - NDQ, which the
                // recompute below reuses)
                if (i >= C::NPART) {
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait_bounded(pempty(pb), ((i / C::NPART) - 1) & 1, abort_flag, p));
                    if (!ok) break;
                }
                // before the recompute below stores its first state (same slot)
                load_rev(lenv - 1);
            }
            if (has_rec) {
                ok = __all_sync(0xffffffffu,
                                mbar_wait_bounded(in_full(m % C::NSTAGE), (m / C::NSTAGE) & 1, abort_flag, p));
                if (!ok) break;
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(ck_full, m & 1, abort_flag, p));
                if (!ok) break;
                const float* ck = reinterpret_cast<const float*>(smem + C::OFF_CK);
#pragma unroll
                for (int r = 0; r < C::RT; ++r) h[r] = jv ? ck[(row0 + r) * V + j] : 0.f;
                __syncwarp();
                if (lane == 0) mbar_arrive(ck_empty);
                if constexpr (C::OC) {
                    put_state_hi<C>(rec_ring, h);
                } else {
                    st_vec(Sst, sslot(m, 0), h);
                    if (jv) write_state_operand_hi<C>(Br, h, j, nloc);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bready_rec(tile));
            }
            auto rev_step = [&](int s) -> bool {
                // ---------------------------------------- reverse step t = c0v + u
                const int u = lenv - 1 - s;
                if (s > 0) {   // fold in dA_{t+1} Wᵀ from the previous reverse step
                    ok = __all_sync(0xffffffffu, mbar_wait_bounded(accfull_rev(tile), nrev & 1, abort_flag, p));
                    if (!ok) return false;
                    ++nrev;
                    tc_fence_after();
                    uint32_t dhi[C::RT], dlo[C::RT];
                    load_acc<C>(tb_rev, dhi, dlo);
                    tc_wait_ld();
                    reg_fence(dhi);
                    reg_fence(dlo);
#pragma unroll
                    for (int r = 0; r < C::RT; ++r)
                        G[r] = fmaf(fprev, G[r], __uint_as_float(dhi[r]) + __uint_as_float(dlo[r]));
                    tc_fence_before();
                } else if constexpr (C::OC) {
                    tc_wait_ld();   // the chunk's first Z's
                }
                if constexpr (C::OC) {
                    reg_fence(szr);
#pragma unroll
                    for (int r = 0; r < C::RT; ++r) zc[r] = __uint_as_float(szr[r]);
                }
                const float dyj = bf16_at(stv, C::ST_DY + (u + 1) * V * 2);
                const float vj = bf16_at(stv, C::ST_V + u * V * 2);
                const float ft = *reinterpret_cast<const float*>(stv + C::ST_F + u * 4);
                float qq[C::RT], kk[C::RT];
                lds_bf16<C::RT>(reinterpret_cast<const uint16_t*>(stv + C::ST_Q + u * K * 2) + row0, qq);
                lds_bf16<C::RT>(reinterpret_cast<const uint16_t*>(stv + C::ST_K + u * K * 2) + row0, kk);
                float dA[C::RT], pk[C::RT];
                float dfp = 0.f, dvp = 0.f;
#pragma unroll
                for (int r = 0; r < C::RT; ++r) {
                    const float z = zc[r];
                    G[r] = fmaf(qq[r], dyj, G[r]);
                    dA[r] = (1.f - ft) * G[r] * fmaf(-z, z, 1.f);
                    dfp = fmaf(G[r], hpc[r] - z, dfp);
                    dvp = fmaf(dA[r], kk[r], dvp);
                    pk[r] = dA[r] * vj;
                }
                if (jv) {
                    write_state_operand<C, true>(Bd, dA, j, nloc);
                    // the dW MMA reads H_{t-1} (hi half only): on chip, from the ring
                    if constexpr (!C::OC) write_dw_a_operand<C>(Bs, hpc, j, nloc);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bready_rev(tile));
                if (u > 0) load_rev(u - 1);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) dfp += __shfl_xor_sync(0xffffffffu, dfp, o);
                if (lane == 0) part[(C::DFP / 4) + u * C::NWE + warp] = dfp;
                if constexpr (C::MX == 64) dvp += __shfl_xor_sync(0xffffffffu, dvp, 16);
                if (half == 0 && jv) part[(C::DVP / 4) + (u * C::NSLOT + slot) * V + j] = dvp;
                // dk_t[i] = Σ_j dA_t[i, j] v_t[j]
                row_sum_store(pk, part + (C::DKP / 4) + u * 4 * K);
                fprev = ft;
                return true;
            };
            auto rec_step = [&](int s) -> bool {
                // ---------------------------------------- recompute step c0r + u
                const int u = s;
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(accfull_rec(tile), nrec & 1, abort_flag, p));
                if (!ok) return false;
                ++nrec;
                tc_fence_after();
                const float vj = bf16_at(str, C::ST_V + u * V * 2);
                const float g = 1.f - *reinterpret_cast<const float*>(str + C::ST_F + u * 4);
                uint32_t ahi[C::RT];
                load_acc_hi<C>(tb_rec, ahi);
                float kk[C::RT];
                lds_bf16<C::RT>(reinterpret_cast<const uint16_t*>(str + C::ST_K + u * K * 2) + row0, kk);
                tc_wait_ld();
                reg_fence(ahi);
                float zz[C::RT];
#pragma unroll
                for (int r = 0; r < C::RT; r += 2) {
                    const float2 z2 = tanh2_ex2(make_float2(fmaf(kk[r], vj, __uint_as_float(ahi[r])),
                                                            fmaf(kk[r + 1], vj, __uint_as_float(ahi[r + 1]))));
                    zz[r] = z2.x;
                    zz[r + 1] = z2.y;
                    h[r] = fmaf(g, z2.x - h[r], h[r]);
                    h[r + 1] = fmaf(g, z2.y - h[r + 1], h[r + 1]);
                }
                if constexpr (C::OC) {
                    uint32_t zb[C::RT];
#pragma unroll
                    for (int r = 0; r < C::RT; ++r) zb[r] = __float_as_uint(zz[r]);
                    tmem_st_32x32b<C::RT>(rec_scr + (uint32_t)(u * rec_sstep), zb);
                } else {
                    st_vec(Sz, sslot(m, u), zz);
                    if (u + 1 < lenr) st_vec(Sst, sslot(m, u + 1), h);   // H_{c0+len} is not read back
                }
                tc_fence_before();
                if (u + 1 < lenr) {
                    if constexpr (C::OC) put_state_hi<C>(rec_ring + (u + 1) * rec_rstep, h);
                    else if (jv) write_state_operand_hi<C>(Br, h, j, nloc);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bready_rec(tile));
                }
                // dq_t[i] = Σ_j H_{t+1}[i, j] dy_t[j] for t = c0r + u (h is H_{t+1} now)
                const float dyj = bf16_at(str, C::ST_DY + (u + 1) * V * 2);
                float pq[C::RT];
#pragma unroll
                for (int r = 0; r < C::RT; ++r) pq[r] = h[r] * dyj;
                row_sum_store(pq, dqp + u * 4 * K);
                return true;
            };
            const int nsteps = max(lenr, lenv);
#pragma unroll 2   // (32.2 -> 31.8 ms at the 7B-MoE training shape)
            for (int s = 0; s < nsteps && ok; ++s) {
                if (s < lenv) ok = rev_step(s);
                if (ok && s < lenr) ok = rec_step(s);
            }
            if (!ok) break;
            if (has_rev) {
                // G_{c0-1} = f_{c0} G_{c0} + dA_{c0} Wᵀ
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(accfull_rev(tile), nrev & 1, abort_flag, p));
                if (!ok) break;
                ++nrev;
                tc_fence_after();
                {
                    uint32_t dhi[C::RT], dlo[C::RT];
                    load_acc<C>(tb_rev, dhi, dlo);
                    tc_wait_ld();
                    reg_fence(dhi);
                    reg_fence(dlo);
#pragma unroll
                    for (int r = 0; r < C::RT; ++r)
                        G[r] = fmaf(fprev, G[r], __uint_as_float(dhi[r]) + __uint_as_float(dlo[r]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(in_empty((m - 1) % C::NSTAGE));
                    mbar_arrive(pfull(pb));
                }
            }
        }
        if constexpr (C::OC) {   // no scratch store or load in flight when the columns are freed
            tc_wait_st();
            tc_wait_ld();
        }
        if (ok && jv) {
#pragma unroll
            for (int r = 0; r < C::RT; ++r) p.dH0[sbase + (size_t)(row0 + r) * V + j] = G[r];
        }
    } else if (warp == C::W_PROD) {
        // ------------------------------------------------------------ producer (chunks in reverse order)
        int last = -1, last_ck = -1;   // last chunk whose inputs / checkpoint were requested
        const int qkb = qk_pair(p, bh);   // k / q rows of this pair's head group
        for (int i = 0; i < nck; ++i) {
            if (p.fault == 1 && i >= 1) break;   // injected: stop feeding the ring after the first chunk
            const int c0 = (nck - 1 - i) * CS, len = min(CS, T - c0), s = i % C::NSTAGE;
            if (i >= C::NSTAGE) {
                const bool ok = __all_sync(
                    0xffffffffu, mbar_wait_bounded(in_empty(s), ((i / C::NSTAGE) - 1) & 1, abort_flag, p));
                if (!ok) break;
            }
            uint8_t* st = smem + C::OFF_RING + s * C::STAGE_BYTES;
            if (lane < len)
                reinterpret_cast<float*>(st + C::ST_F)[lane] = gate_value(p, p.f[(size_t)bh * T + c0 + lane]);
            __syncwarp();
            const size_t rk = ((size_t)qkb * T + c0) * KF + koff, rv = ((size_t)bh * T + c0) * V;
            if (lane == 0) {
                const uint32_t kb = (uint32_t)(len * K * 2), vb = (uint32_t)(len * V * 2);
                // dy rows c0-1 .. c0+len-1; the row of step c0-1 exists only when c0 > 0
                const uint32_t dyb = (uint32_t)((len + (c0 > 0 ? 1 : 0)) * V * 2);
                mbar_arrive_expect_tx(in_full(s), 2 * kb + vb + dyb);
                const uint16_t* dyg = static_cast<const uint16_t*>(p.dy) + rv;
                if (nsl == 1) {
                    bulk_g2s(smem_u32(st + C::ST_K), static_cast<const uint16_t*>(p.k) + rk, kb, in_full(s));
                    bulk_g2s(smem_u32(st + C::ST_Q), static_cast<const uint16_t*>(p.q) + rk, kb, in_full(s));
                }
                bulk_g2s(smem_u32(st + C::ST_V), static_cast<const uint16_t*>(p.v) + rv, vb, in_full(s));
                if (c0 > 0)
                    bulk_g2s(smem_u32(st + C::ST_DY), dyg - V, dyb, in_full(s));
                else
                    bulk_g2s(smem_u32(st + C::ST_DY + V * 2), dyg, dyb, in_full(s));
            }
            if (nsl > 1) {
                // this slice's K values of each step's k and q row (strided in HBM)
                __syncwarp();
                if (lane < len) {
                    const size_t r = rk + (size_t)lane * KF;
                    bulk_g2s(smem_u32(st + C::ST_K + lane * K * 2), static_cast<const uint16_t*>(p.k) + r, K * 2,
                             in_full(s));
                    bulk_g2s(smem_u32(st + C::ST_Q + lane * K * 2), static_cast<const uint16_t*>(p.q) + r, K * 2,
                             in_full(s));
                }
            }
            last = i;
            // checkpoint H_{c0} of this slice, once every warp has read the previous one
            if (i >= 1) {
                const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(ck_empty, (i - 1) & 1, abort_flag, p));
                if (!ok) break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(ck_full, (uint32_t)(K * V * 4));
                const float* ck = p.ckpt + ((size_t)bh * nck + (nck - 1 - i)) * KF * V + (size_t)koff * V;
                bulk_g2s(smem_u32(smem + C::OFF_CK), ck, (uint32_t)(K * V * 4), ck_full);
            }
            last_ck = i;
        }
        // on an abort, copies may still be in flight: wait for them (bounded)
        // before the CTA's shared memory is released
        if (lane == 0) {
            for (int i = max(0, last - (C::NSTAGE - 1)); i <= last; ++i)
                mbar_wait_drain(in_full(i % C::NSTAGE), (i / C::NSTAGE) & 1, p);
            if (last_ck >= 0) mbar_wait_drain(ck_full, last_ck & 1, p);
        }
        __syncwarp();
    } else if (warp == C::W_MREV) {
        // ------------------------------------------------------------ MMA issuer: reverse chain
        if (lane == 0) {
            constexpr uint32_t idesc_g = idesc_bf16_f32(C::MX, C::NT, 1, 1);
            constexpr uint32_t idesc_w = idesc_bf16_f32(C::MX, V, 0, 0);
            const uint32_t w0 = smem_u32(smem + C::OFF_W);
            uint32_t nbr[C::P];
            int issued[C::P];
#pragma unroll
            for (int i = 0; i < C::P; ++i) {
                nbr[i] = 0;
                issued[i] = -1;
            }
            bool first_dw = true, ok = true;
            for (int i = 0; i < nck && ok; ++i) {
                const int len = min(CS, T - (nck - 1 - i) * CS);
                for (int u = 0; u < len && ok; ++u) {
#pragma unroll
                    for (int tile = 0; tile < C::P; ++tile) {
                        if (!mbar_wait_bounded(bready_rev(tile), nbr[tile] & 1, abort_flag, p)) {
                            ok = false;
                            break;
                        }
                        ++nbr[tile];
                        tc_fence_after();
                        // H_{t-1} of reverse step u: on chip, the ring slot of chunk step len-1-u
                        const int us = len - 1 - u;
                        const uint32_t bs = smem_u32(
                            smem + (C::OC ? C::OFF_BR + (((i & 1) ? CS + 1 - us : us) * C::P + tile) * C::BS_BYTES
                                          : C::OFF_BS + tile * C::BS_BYTES));
                        const uint32_t bd = smem_u32(smem + C::OFF_BD + tile * C::B_BYTES);
                        const uint32_t dt = tmem + (uint32_t)(C::REV_COL + tile * C::NT);
                        // G-propagation: A = W (MN-major view of the shared W buffer)
#pragma unroll
                        for (int ks = 0; ks < V / 16; ++ks)
                            tc_mma_f16_ss(dt, smem_desc(w0 + ks * 2 * C::MX * 16, C::MX * 16, 128),
                                          smem_desc(bd + ks * 2 * C::NT * 16, C::NT * 16, 128), idesc_g,
                                          ks > 0 ? 1u : 0u);
                        // dW += H_{t-1}ᵀ dA_t over the tile's rows (16 per k-step)
#pragma unroll
                        for (int ks = 0; ks < C::R / 16; ++ks)
                            tc_mma_f16_ss(tmem + C::DW_COL, smem_desc(bs + ks * 256, 128, C::R * 16),
                                          smem_desc(bd + ks * 256, 128, C::NT * 16), idesc_w,
                                          (first_dw && ks == 0) ? 0u : 1u);
                        first_dw = false;
                        tc_commit(accfull_rev(tile));
                        issued[tile] = (int)(nbr[tile] - 1);
                    }
                }
            }
#pragma unroll
            for (int tile = 0; tile < C::P; ++tile)
                if (issued[tile] >= 0) mbar_wait_drain(accfull_rev(tile), (uint32_t)issued[tile] & 1, p);
        }
        __syncwarp();
    } else if (warp == C::W_MREC) {
        // ------------------------------------------------------------ MMA issuer: recompute chain
        if (lane == 0) {
            constexpr uint32_t idesc_f = idesc_bf16_f32(C::MX, C::R, 0, 1);   // the state's hi half only
            const uint32_t w0 = smem_u32(smem + C::OFF_W);
            uint32_t nbr[C::P];
            int issued[C::P];
#pragma unroll
            for (int i = 0; i < C::P; ++i) {
                nbr[i] = 0;
                issued[i] = -1;
            }
            bool ok = true;
            for (int i = 0; i < nck && ok; ++i) {
                const int nm = min(CS, T - (nck - 1 - i) * CS);
                for (int u = 0; u < nm && ok; ++u) {
#pragma unroll
                    for (int tile = 0; tile < C::P; ++tile) {
                        if (!mbar_wait_bounded(bready_rec(tile), nbr[tile] & 1, abort_flag, p)) {
                            ok = false;
                            break;
                        }
                        ++nbr[tile];
                        tc_fence_after();
                        // the state operand: on chip, the ring slot of chunk step u (R rows)
                        constexpr int NB = C::OC ? C::R : C::NT;
                        const uint32_t br = smem_u32(
                            smem + (C::OC ? C::OFF_BR + (((i & 1) ? CS + 1 - u : u) * C::P + tile) * C::BS_BYTES
                                          : C::OFF_BR + tile * C::B_BYTES));
                        const uint32_t dt = tmem + (uint32_t)(C::REC_COL + tile * C::NT);
                        // recompute: A = Wᵀ (K-major view of the shared W buffer)
#pragma unroll
                        for (int ks = 0; ks < V / 16; ++ks)
                            tc_mma_f16_ss(dt, smem_desc(w0 + ks * 256, 128, C::MX * 16),
                                          smem_desc(br + ks * 2 * NB * 16, NB * 16, 128), idesc_f,
                                          ks > 0 ? 1u : 0u);
                        tc_commit(accfull_rec(tile));
                        issued[tile] = (int)(nbr[tile] - 1);
                    }
                }
            }
#pragma unroll
            for (int tile = 0; tile < C::P; ++tile)
                if (issued[tile] >= 0) mbar_wait_drain(accfull_rec(tile), (uint32_t)issued[tile] & 1, p);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ storer: dv, df, dk, dq
        float* const dv_out = nsl == 1 ? p.dv : p.dv_part + (size_t)sl * p.B * p.H * T * V;
        float* const df_out = nsl == 1 ? p.df : p.df_part + (size_t)sl * p.B * p.H * T;
        for (int i = 0; i < nck; ++i) {
            const int c0 = (nck - 1 - i) * CS, len = min(CS, T - c0), b = i % C::NPART;
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(pfull(b), (i / C::NPART) & 1, abort_flag, p));
            if (!ok) break;
            const float* part = reinterpret_cast<const float*>(smem + C::OFF_PART + b * C::PART_BYTES);
            const float* dqp = reinterpret_cast<const float*>(smem + C::OFF_DQ + (i % C::NDQ) * C::DQ_BYTES);
            for (int e = lane; e < len * V; e += 32) {
                const int u = e / V, jj = e % V;
                float sv = 0.f;
#pragma unroll
                for (int s = 0; s < C::NSLOT; ++s) sv += part[C::DVP / 4 + (u * C::NSLOT + s) * V + jj];
                dv_out[((size_t)bh * T + c0 + u) * V + jj] = sv;
            }
            if (lane < len) {
                float sf = 0.f;
#pragma unroll
                for (int w = 0; w < C::NWE; ++w) sf += part[C::DFP / 4 + lane * C::NWE + w];
                // per slice: the chain rule through the logistic gate is linear
                df_out[(size_t)bh * T + c0 + lane] = gate_grad(p, p.f[(size_t)bh * T + c0 + lane], sf);
            }
            for (int e = lane; e < len * K; e += 32) {
                const int u = e / K, rr = e % K;
                const float* pk = part + C::DKP / 4 + u * 4 * K + rr;
                const float* pq = dqp + u * 4 * K + rr;
                const size_t o = ((size_t)bh * T + c0 + u) * KF + koff + rr;
                p.dk[o] = ((pk[0] + pk[K]) + pk[2 * K]) + pk[3 * K];
                p.dq[o] = ((pq[0] + pq[K]) + pq[2 * K]) + pq[3 * K];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(pempty(b));
        }
    }

    // dW partial of this CTA: TMEM row l (of MX) holds row l of Σ H_{t-1}ᵀ dA_t
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp < 4 && *abort_flag == 0) {
        if constexpr (C::MX == 64) {
            constexpr int H2 = V / 2;   // columns per half-warp
            uint32_t w[H2];
            tmem_ld_16x32bx2<H2, H2>(tmem + ((uint32_t)(warp * 32) << 16) + C::DW_COL, w);
            tc_wait_ld();
            reg_fence(w);
            const int l = warp * 16 + (lane & 15), j0 = (lane >> 4) * H2;
            if (l < V) {
                float* dst = p.dW_part + ((size_t)blockIdx.x * V + l) * V + j0;
#pragma unroll
                for (int e = 0; e < H2; e += 4)
                    *reinterpret_cast<float4*>(dst + e) = make_float4(
                        __uint_as_float(w[e]), __uint_as_float(w[e + 1]), __uint_as_float(w[e + 2]),
                        __uint_as_float(w[e + 3]));
            }
        } else {
            const int l = warp * 32 + lane;
#pragma unroll
            for (int c0 = 0; c0 < V; c0 += 32) {
                uint32_t w[32];
                tmem_ld_32x32b<32>(tmem + ((uint32_t)(warp * 32) << 16) + C::DW_COL + c0, w);
                tc_wait_ld();
                reg_fence(w);
                float* dst = p.dW_part + ((size_t)blockIdx.x * V + l) * V + c0;
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4*>(dst + e) = make_float4(
                        __uint_as_float(w[e]), __uint_as_float(w[e + 1]), __uint_as_float(w[e + 2]),
                        __uint_as_float(w[e + 3]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == C::W_PROD) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// dv = Σ_s dv_part[s] and df = Σ_s df_part[s] over the slices, in slice order.
__global__ void m2rnn_slice_sum_kernel(const Params p) {
    const size_t ndv = (size_t)p.B * p.H * p.T * p.V, ndf = (size_t)p.B * p.H * p.T;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < ndv + ndf; e += (size_t)gridDim.x * blockDim.x) {
        const bool dv = e < ndv;
        const size_t o = dv ? e : e - ndv, n = dv ? ndv : ndf;
        const float* src = (dv ? p.dv_part : p.df_part) + o;
        float s = src[0];
        for (int sl = 1; sl < p.slices; ++sl) s += src[(size_t)sl * n];
        (dv ? p.dv : p.df)[o] = s;
    }
}

namespace {

// Slice rows: V = 128 takes at most 32 rows per CTA (8 rows per thread), the
// narrower states at most 64.
int tcg_slice_rows(int K, int V) {
    const int cap = V == 128 ? 32 : 64;
    return K < cap ? K : cap;
}

// The chunk stays on chip for V = 128 when tensor memory holds C steps.
template <int KS, int V>
bool tcg_on_chip(int C) {
    if constexpr (V == 128) return C <= BwdTcgCfg<KS, V, true>::CMAX;
    return false;
}

template <int KS, int V, bool OC>
cudaError_t launch_tcg(const Params& p0, cudaStream_t stream) {
    using C = BwdTcgCfg<KS, V, OC>;
    Params p = p0;
    p.slices = p.K / KS;
    p.dw_parts = p.slices;   // one dW partial per slice
    const size_t ncta = (size_t)p.B * p.H * p.slices;
    p.dv_part = p.scratch + (OC ? 0 : 2 * (size_t)p.C * ncta * KS * C::MX);
    p.df_part = p.dv_part + (size_t)p.slices * p.B * p.H * p.T * V;
    auto kern = m2rnn_bwd_tcg_kernel<KS, V, OC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)ncta, C::NTHREADS, C::SMEM_BYTES, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.slices > 1) {
        const size_t n = (size_t)p.B * p.H * p.T * (V + 1);
        const size_t want = (n + 255) / 256, cap = (size_t)kNumSMs * 8;
        m2rnn_slice_sum_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, stream>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_dw_reduce(p, stream);
}

template <int KS, int V>
cudaError_t launch_tcg_ks(const Params& p, cudaStream_t s) {
    if constexpr (V == 128)
        if (tcg_on_chip<KS, V>(p.C)) return launch_tcg<KS, V, true>(p, s);
    return launch_tcg<KS, V, false>(p, s);
}

template <int V>
cudaError_t launch_tcg_v(const Params& p, cudaStream_t s) {
    switch (tcg_slice_rows(p.K, V)) {
        case 16: return launch_tcg_ks<16, V>(p, s);
        case 32: return launch_tcg_ks<32, V>(p, s);
        case 64:
            if constexpr (V <= 64) return launch_tcg_ks<64, V>(p, s);
            break;
    }
    return cudaErrorNotSupported;
}

bool tcg_chunk_on_chip(int K, int V, int C) {
    if (V != 128) return false;
    return tcg_slice_rows(K, V) == 16 ? tcg_on_chip<16, 128>(C) : tcg_on_chip<32, 128>(C);
}

}  // namespace

int bwd_tcg_slices(int K, int V) { return K / tcg_slice_rows(K, V); }

bool bwd_tcg_supported(int K, int V, int C) {
    const bool kv = (K == 16 || K == 32 || K == 64 || K == 128) && (V == 16 || V == 32 || V == 64 || V == 128);
    return kv && C >= 1 && C <= BwdTcgCfg<16, 16>::CMAX;
}

// Per CTA: a dW partial and, unless the chunk stays on chip, 2·C·KS·MX
// scratch values; with several slices per pair, the slices' dv and df partials.
size_t bwd_tcg_workspace(int B, int H, int T, int K, int V, int C) {
    if (!bwd_tcg_supported(K, V, C)) return 0;
    const size_t ks = (size_t)tcg_slice_rows(K, V), nsl = (size_t)K / ks, mx = V <= 64 ? 64 : 128;
    const size_t ncta = (size_t)B * H * nsl;
    size_t n = ncta * V * V + (tcg_chunk_on_chip(K, V, C) ? 0 : 2 * (size_t)C * ncta * ks * mx);
    if (nsl > 1) n += nsl * (size_t)B * H * T * (V + 1);
    return sizeof(float) * n;
}

cudaError_t launch_bwd_tcg(const Params& p, cudaStream_t s) {
    if (!bwd_tcg_supported(p.K, p.V, p.C)) return cudaErrorNotSupported;
    switch (p.V) {
        case 16: return launch_tcg_v<16>(p, s);
        case 32: return launch_tcg_v<32>(p, s);
        case 64: return launch_tcg_v<64>(p, s);
        case 128: return launch_tcg_v<128>(p, s);
    }
    return cudaErrorNotSupported;
}

}  // namespace m2rnn
