// C ABI of libm2rnn.so: argument validation, workspace carving and dispatch
// to the kernels.  The operation and the tensor layouts are documented in
// include/m2rnn.h.
#include <atomic>
#include <cstdint>
#include <cstring>

#include "../../include/m2rnn.h"
#include "kernels.h"

namespace {

std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
std::atomic<int> g_fault{0};
constexpr size_t kStatusBytes = 256;

bool shape_ok(int n) { return n == 16 || n == 32 || n == 64 || n == 128; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

m2rnn_status check_dims(const m2rnn_dims* d) {
    if (d == nullptr) return M2RNN_ERR_INVALID_ARG;
    if (d->B < 0 || d->H < 0 || d->T < 0) return M2RNN_ERR_INVALID_ARG;
    if (d->mode < M2RNN_MODE_BF16_TC || d->mode > M2RNN_MODE_BF16_MMA_SYNC) return M2RNN_ERR_INVALID_ARG;
    // k / q head groups: 0 = one per head, else a divisor of H
    if (d->qk_heads < 0 || (d->qk_heads > 0 && (d->qk_heads > d->H || d->H % d->qk_heads != 0)))
        return M2RNN_ERR_INVALID_ARG;
    if (d->f_is_logit != 0 && d->f_is_logit != 1) return M2RNN_ERR_INVALID_ARG;
    if (!shape_ok(d->K) || !shape_ok(d->V) || d->ckpt_stride < 1) return M2RNN_ERR_UNSUPPORTED_SHAPE;
    return M2RNN_OK;
}

int qk_groups(const m2rnn_dims* d) { return d->qk_heads > 0 ? d->qk_heads : d->H; }

// Backward with grouped k / q: per-head dk and dq (fp32 [B][H][T][K] each)
// before the sum over each group's heads.
size_t qk_group_partial_bytes(const m2rnn_dims* d) {
    if (qk_groups(d) == d->H) return 0;
    return 2 * sizeof(float) * (size_t)d->B * d->H * d->T * d->K;
}

m2rnn::Params base_params(const m2rnn_dims* d, void* ws) {
    m2rnn::Params p;
    std::memset(&p, 0, sizeof p);
    p.B = d->B; p.H = d->H; p.T = d->T; p.K = d->K; p.V = d->V; p.C = d->ckpt_stride;
    p.G = qk_groups(d);
    p.f_is_logit = d->f_is_logit;
    p.status = static_cast<uint32_t*>(ws);
    p.wait_limit_ns = g_wait_limit_ns.load();
    p.fault = g_fault.load();
    p.dw_parts = 1;
    p.slices = 1;
    return p;
}

}  // namespace

extern "C" {

size_t m2rnn_workspace_size(const m2rnn_dims* d, int backward) {
    if (check_dims(d) != M2RNN_OK) return 0;
    size_t n = kStatusBytes;
    if (backward && (d->mode == M2RNN_MODE_BF16_TC_FAST_TANH || d->mode == M2RNN_MODE_BF16_MMA_SYNC))
        return 0;   // forward-only modes
    if (!backward && (d->mode == M2RNN_MODE_BF16_TC || d->mode == M2RNN_MODE_BF16_TC_FAST_TANH)) {
        // partial readouts of sliced rows
        const int sl = m2rnn::fwd_tc_slices(d->B, d->H, d->K, d->V);
        if (sl > 1) n += sizeof(float) * (size_t)sl * d->B * d->H * d->T * d->V;
    }
    if (backward) {
        const size_t extra = d->mode == M2RNN_MODE_FP32_DEBUG
                                 ? m2rnn::bwd_fp32_workspace(d->B, d->H, d->K, d->V, d->ckpt_stride)
                                 : m2rnn::bwd_tc_workspace(d->B, d->H, d->T, d->K, d->V, d->ckpt_stride);
        n += (extra + 255) / 256 * 256;
        n += qk_group_partial_bytes(d);
    }
    return n;
}

m2rnn_status m2rnn_forward(const m2rnn_dims* d, const void* k, const void* v, const void* q, const float* f,
                           const void* W, const float* H0, float* y, float* HT, float* ckpt, void* workspace,
                           size_t ws_bytes, m2rnn_stream_t stream) {
    m2rnn_status st = check_dims(d);
    if (st != M2RNN_OK) return st;
    // A tensor with no elements may be passed as NULL.
    const bool seq = (long long)d->B * d->H * d->T > 0;
    if ((seq && (!k || !v || !q || !f || !y)) || (d->H > 0 && !W) || !workspace) return M2RNN_ERR_INVALID_ARG;
    const void* ptrs[] = {k, v, q, f, W, H0, y, HT, ckpt, workspace};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return M2RNN_ERR_MISALIGNED;
    if (ws_bytes < m2rnn_workspace_size(d, 0)) return M2RNN_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((long long)d->B * d->H == 0) return M2RNN_OK;
    const size_t state_bytes = sizeof(float) * (size_t)d->B * d->H * d->K * d->V;
    if (d->T == 0) {   // no steps: H_T = H0
        if (HT) {
            cudaError_t e = H0 ? (H0 == HT ? cudaSuccess   // in place: nothing to do
                                           : cudaMemcpyAsync(HT, H0, state_bytes, cudaMemcpyDeviceToDevice, s))
                               : cudaMemsetAsync(HT, 0, state_bytes, s);
            if (e != cudaSuccess) return M2RNN_ERR_CUDA;
        }
        return M2RNN_OK;
    }
    m2rnn::Params p = base_params(d, workspace);
    p.k = k; p.v = v; p.q = q; p.f = f; p.W = W; p.H0 = H0; p.y = y; p.HT = HT; p.ckpt = ckpt;
    p.ypart = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kStatusBytes);
    p.fast_tanh = d->mode == M2RNN_MODE_BF16_TC_FAST_TANH;
    cudaError_t e = d->mode == M2RNN_MODE_FP32_DEBUG    ? m2rnn::launch_fwd_fp32(p, s)
                    : d->mode == M2RNN_MODE_BF16_MMA_SYNC ? m2rnn::launch_fwd_mma(p, s)
                                                          : m2rnn::launch_fwd_tc(p, s);
    if (e == cudaErrorNotSupported) return M2RNN_ERR_UNSUPPORTED_SHAPE;
    return e == cudaSuccess ? M2RNN_OK : M2RNN_ERR_CUDA;
}

m2rnn_status m2rnn_backward(const m2rnn_dims* d, const void* k, const void* v, const void* q, const float* f,
                            const void* W, const float* ckpt, const void* dy, const float* dHT, float* dk, float* dv,
                            float* dq, float* df, float* dW, float* dH0, void* workspace, size_t ws_bytes,
                            m2rnn_stream_t stream) {
    m2rnn_status st = check_dims(d);
    if (st != M2RNN_OK) return st;
    if (d->mode == M2RNN_MODE_BF16_TC_FAST_TANH || d->mode == M2RNN_MODE_BF16_MMA_SYNC)
        return M2RNN_ERR_INVALID_ARG;   // forward-only modes
    // A tensor with no elements may be passed as NULL.
    const bool seq = (long long)d->B * d->H * d->T > 0;
    const bool state = (long long)d->B * d->H > 0;
    if ((seq && (!k || !v || !q || !f || !dy || !dk || !dv || !dq || !df || !ckpt)) || (d->H > 0 && (!W || !dW)) ||
        (state && !dH0) || !workspace)
        return M2RNN_ERR_INVALID_ARG;
    if (d->mode == M2RNN_MODE_BF16_TC && !m2rnn::bwd_tc_supported(d->K, d->V, d->ckpt_stride))
        return M2RNN_ERR_UNSUPPORTED_SHAPE;
    const void* ptrs[] = {k, v, q, f, W, ckpt, dy, dHT, dk, dv, dq, df, dW, dH0, workspace};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return M2RNN_ERR_MISALIGNED;
    if (ws_bytes < m2rnn_workspace_size(d, 1)) return M2RNN_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t wbytes = sizeof(float) * (size_t)d->H * d->V * d->V;
    if ((long long)d->B * d->H == 0) {
        if (wbytes && cudaMemsetAsync(dW, 0, wbytes, s) != cudaSuccess) return M2RNN_ERR_CUDA;
        return M2RNN_OK;
    }
    if (d->T == 0) {   // no steps: dH0 = dHT, dW = 0
        const size_t state_bytes = sizeof(float) * (size_t)d->B * d->H * d->K * d->V;
        cudaError_t e = dHT ? (dHT == dH0 ? cudaSuccess
                                          : cudaMemcpyAsync(dH0, dHT, state_bytes, cudaMemcpyDeviceToDevice, s))
                            : cudaMemsetAsync(dH0, 0, state_bytes, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(dW, 0, wbytes, s);
        return e == cudaSuccess ? M2RNN_OK : M2RNN_ERR_CUDA;
    }
    m2rnn::Params p = base_params(d, workspace);
    p.k = k; p.v = v; p.q = q; p.f = f; p.W = W; p.ckpt = const_cast<float*>(ckpt);
    p.dy = dy; p.dHT = dHT; p.dk = dk; p.dv = dv; p.dq = dq; p.df = df; p.dW = dW; p.dH0 = dH0;
    uint8_t* extra = static_cast<uint8_t*>(workspace) + kStatusBytes;
    p.dW_part = reinterpret_cast<float*>(extra);
    p.dw_parts = d->mode == M2RNN_MODE_FP32_DEBUG ? 1 : m2rnn::bwd_tc_slices(d->K, d->V, d->ckpt_stride);
    p.scratch = p.dW_part + (size_t)d->B * d->H * p.dw_parts * d->V * d->V;
    const bool grouped = qk_group_partial_bytes(d) != 0;
    if (grouped) {   // the kernels write per-head dk / dq here; the group sums go to dk, dq
        const size_t extra_bytes = d->mode == M2RNN_MODE_FP32_DEBUG
                                       ? m2rnn::bwd_fp32_workspace(d->B, d->H, d->K, d->V, d->ckpt_stride)
                                       : m2rnn::bwd_tc_workspace(d->B, d->H, d->T, d->K, d->V, d->ckpt_stride);
        p.dk = reinterpret_cast<float*>(extra + (extra_bytes + 255) / 256 * 256);
        p.dq = p.dk + (size_t)d->B * d->H * d->T * d->K;
    }
    cudaError_t e = d->mode == M2RNN_MODE_FP32_DEBUG ? m2rnn::launch_bwd_fp32(p, s) : m2rnn::launch_bwd_tc(p, s);
    if (e == cudaSuccess && grouped) e = m2rnn::launch_qk_group_reduce(p, p.dk, p.dq, dk, dq, s);
    if (e == cudaErrorNotSupported) return M2RNN_ERR_UNSUPPORTED_SHAPE;
    return e == cudaSuccess ? M2RNN_OK : M2RNN_ERR_CUDA;
}

m2rnn_status m2rnn_get_device_status(void* workspace, m2rnn_stream_t stream) {
    if (!workspace) return M2RNN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return M2RNN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return M2RNN_ERR_CUDA;
    if (word != 0) {
        if (cudaMemsetAsync(workspace, 0, sizeof word, s) != cudaSuccess) return M2RNN_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return M2RNN_ERR_CUDA;
        return M2RNN_ERR_DEVICE_TIMEOUT;
    }
    return M2RNN_OK;
}

const char* m2rnn_status_string(m2rnn_status s) {
    switch (s) {
        case M2RNN_OK: return "M2RNN_OK";
        case M2RNN_ERR_INVALID_ARG: return "M2RNN_ERR_INVALID_ARG";
        case M2RNN_ERR_UNSUPPORTED_SHAPE: return "M2RNN_ERR_UNSUPPORTED_SHAPE";
        case M2RNN_ERR_MISALIGNED: return "M2RNN_ERR_MISALIGNED";
        case M2RNN_ERR_WORKSPACE: return "M2RNN_ERR_WORKSPACE";
        case M2RNN_ERR_CUDA: return "M2RNN_ERR_CUDA";
        case M2RNN_ERR_DEVICE_TIMEOUT: return "M2RNN_ERR_DEVICE_TIMEOUT";
    }
    return "M2RNN_ERR_UNKNOWN";
}

void m2rnn_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns < 100000ull ? 100000ull : ns); }

int m2rnn_debug_set_fault(int fault) {
    if (fault != 0 && fault != 1) return M2RNN_ERR_INVALID_ARG;
    g_fault.store(fault);
    return M2RNN_OK;
}

}  // extern "C"
