// Shared device-side pieces of the M²RNN kernels: launch parameters, the
// device status word and bounded mbarrier waits.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace m2rnn {

// Device status codes written into the workspace status word.
enum : uint32_t {
    kDevOk = 0,
    kDevTimeout = 1u,
};

struct Params {
    int B, H, T, K, V, C;
    int G;              // head groups of k and q (G divides H; G == H: one per head)
    int f_is_logit;     // f holds gate logits a_t, f_t = 1 / (1 + exp(-a_t)); df is then dL/da_t
    const void* k;
    const void* v;
    const void* q;
    const float* f;
    const void* W;
    const float* H0;    // forward: initial state (may be null)
    float* y;
    float* HT;          // may be null
    float* ckpt;        // forward: checkpoint output (may be null); backward: input
    // backward
    const void* dy;
    const float* dHT;   // may be null
    float* dk;
    float* dv;
    float* dq;
    float* df;
    float* dW;
    float* dH0;
    float* dW_part;     // [B*H][dw_parts][V][V] partial dW (workspace)
    int dw_parts;       // dW partials per (b, h)
    int slices;         // forward: CTAs (row slices) per (b, h)
    int fast_tanh;      // forward: tanh.approx.f32 instead of the exp-based tanh
    float* ypart;       // forward with slices > 1: [slices][B*H][T][V] partial readouts (workspace)
    float* scratch;     // per-CTA recompute scratch (workspace)
    float* dv_part;     // backward with slices > 1 (general-shape kernel): [slices][B*H][T][V] (workspace)
    float* df_part;     // same: [slices][B*H][T] (workspace)
    uint32_t* status;   // device status word (workspace)
    uint64_t wait_limit_ns;
    int fault;          // injected fault (m2rnn_debug_set_fault), 0 = none
};

// Row block of k and q that pair bh = b·H + h reads: head h uses group
// h / (H/G) of batch element b.  The identity when G == H.
__host__ __device__ __forceinline__ int qk_pair(const Params& p, int bh) {
    return (bh / p.H) * p.G + (bh % p.H) / (p.H / p.G);
}

// Gate f_t from the f input: the value itself, or the logistic function of a
// gate logit (accurate expf and IEEE division; saturates to exactly 0 or 1).
__device__ __forceinline__ float gate_value(const Params& p, float x) {
    return p.f_is_logit ? 1.f / (1.f + expf(-x)) : x;
}

// dL/df_t -> the gradient of the f input: unchanged, or dL/da_t = dL/df_t · f_t (1 - f_t).
__device__ __forceinline__ float gate_grad(const Params& p, float x, float df) {
    if (!p.f_is_logit) return df;
    const float ft = gate_value(p, x);
    return df * (ft * (1.f - ft));
}

// Bounded wait on an mbarrier phase.  Returns false (and raises the CTA-wide
// abort flag and the device status word) when the wait runs longer than the
// limit, or when another thread of the CTA has already aborted.
// SPIN = true polls with test_wait (no suspension: lowest wake-up latency,
// but the waiting warp keeps issuing).
template <bool SPIN = false>
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  const Params& p) {
    if (SPIN ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (SPIN ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > p.wait_limit_ns) {
            *abort_flag = 1;
            atomicOr(p.status, kDevTimeout);
            return false;
        }
    }
}

// Same, but ignores the abort flag (used to drain copies/MMAs in flight
// before the CTA exits).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, const Params& p) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > p.wait_limit_ns) {
            atomicOr(p.status, kDevTimeout);
            return false;
        }
    }
    return true;
}

}  // namespace m2rnn
