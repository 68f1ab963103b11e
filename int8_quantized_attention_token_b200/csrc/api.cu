// api.cu -- the whole-path entry points of libintfa (quantise Q/K per token,
// V per head, then the fused attention; and the same from host buffers) and
// the status strings.  See include/intfa.h for the contract of each call.
#include "internal.h"

namespace {

struct Layout {
    size_t q, k, vt, sq, sk, sv, ws, end;       // device workspace of intfa_forward
    size_t hq, hk, hv, ho, host_end;           // + fp16 staging for intfa_forward_host
};

bool make_layout(int B, int H, int L, int d, Layout *lo) {
    if (B <= 0 || H <= 0 || L <= 0 || (d != 64 && d != 128)) return false;
    const size_t bh = static_cast<size_t>(B) * H;
    if (bh > (1u << 24) || L > 131072) return false;
    const size_t n = bh * static_cast<size_t>(L);              // token rows
    const size_t ld = static_cast<size_t>(intfa_vt_ld(L));
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = intfa::round_up(off + bytes, 256);
        return at;
    };
    lo->q = take(n * d);
    lo->k = take(n * d);
    lo->vt = take(bh * d * ld);
    lo->sq = take(n * sizeof(float));
    lo->sk = take(n * sizeof(float));
    lo->sv = take(bh * sizeof(float));
    lo->ws = take(intfa_quantize_per_tensor_workspace_size(static_cast<int64_t>(bh)));
    lo->end = off;
    lo->hq = take(n * d * 2);
    lo->hk = take(n * d * 2);
    lo->hv = take(n * d * 2);
    lo->ho = take(n * d * 2);
    lo->host_end = off;
    return true;
}

}  // namespace

extern "C" const char *intfa_status_string(int status) {
    switch (status) {
        case INTFA_OK: return "ok";
        case INTFA_ERR_INVALID_ARG: return "invalid argument";
        case INTFA_ERR_UNSUPPORTED: return "unsupported shape";
        case INTFA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case INTFA_ERR_CUDA: return "CUDA call failed";
        case INTFA_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded wait";
        case INTFA_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

extern "C" size_t intfa_forward_workspace_size(int B, int H, int L, int d) {
    Layout lo;
    return make_layout(B, H, L, d, &lo) ? lo.end : 0;
}

extern "C" size_t intfa_forward_host_workspace_size(int B, int H, int L, int d) {
    Layout lo;
    return make_layout(B, H, L, d, &lo) ? lo.host_end : 0;
}

extern "C" int intfa_forward_workspace_layout(int B, int H, int L, int d, size_t offsets[6]) {
    Layout lo;
    if (!offsets || !make_layout(B, H, L, d, &lo)) return INTFA_ERR_INVALID_ARG;
    offsets[0] = lo.q;
    offsets[1] = lo.k;
    offsets[2] = lo.vt;
    offsets[3] = lo.sq;
    offsets[4] = lo.sk;
    offsets[5] = lo.sv;
    return INTFA_OK;
}

extern "C" int intfa_forward(const void *Q_f16, const void *K_f16, const void *V_f16, int B, int H,
                             int L, int d, int causal, void *O_f16, void *workspace,
                             size_t workspace_bytes, void *stream) {
    using namespace intfa;
    Layout lo;
    if (!make_layout(B, H, L, d, &lo)) {
        if (B <= 0 || H <= 0 || L <= 0) return INTFA_ERR_INVALID_ARG;
        return INTFA_ERR_UNSUPPORTED;
    }
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    if (!Q_f16 || !K_f16 || !V_f16 || !O_f16) return INTFA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < lo.end) return INTFA_ERR_WORKSPACE;
    if (!aligned16(Q_f16) || !aligned16(K_f16) || !aligned16(V_f16) || !aligned16(O_f16) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return INTFA_ERR_MISALIGNED;
    uint8_t *w = static_cast<uint8_t *>(workspace);
    int8_t *k = reinterpret_cast<int8_t *>(w + lo.k);
    int8_t *vt = reinterpret_cast<int8_t *>(w + lo.vt);
    float *sq = reinterpret_cast<float *>(w + lo.sq);
    float *sk = reinterpret_cast<float *>(w + lo.sk);
    float *sv = reinterpret_cast<float *>(w + lo.sv);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t rows = static_cast<int64_t>(B) * H * L;
    const int64_t bh = static_cast<int64_t>(B) * H;
    // Q in its own pass: quantising it inside the attention kernel
    // (intfa_attention_fwd_q16) saves the pass but costs more issue slots on
    // the attention kernel's sub-partitions than the pass takes.
    int8_t *q = reinterpret_cast<int8_t *>(w + lo.q);
    int rc = launch_quantize_per_token(Q_f16, rows, d, q, sq, s);
    if (!rc) rc = launch_quantize_per_token(K_f16, rows, d, k, sk, s);
    if (!rc) rc = launch_quantize_per_tensor(V_f16, bh, L, d, 1, vt, sv, w + lo.ws, s);
    if (!rc) rc = launch_attention_fwd(q, k, vt, sq, sk, sv, B, H, L, d, causal, O_f16, s);
    return rc;
}

extern "C" int intfa_forward_host(const void *Q_f16_host, const void *K_f16_host,
                                  const void *V_f16_host, int B, int H, int L, int d, int causal,
                                  void *O_f16_host, void *workspace, size_t workspace_bytes,
                                  void *stream) {
    using namespace intfa;
    Layout lo;
    if (!make_layout(B, H, L, d, &lo)) {
        if (B <= 0 || H <= 0 || L <= 0) return INTFA_ERR_INVALID_ARG;
        return INTFA_ERR_UNSUPPORTED;
    }
    if (!Q_f16_host || !K_f16_host || !V_f16_host || !O_f16_host) return INTFA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < lo.host_end) return INTFA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return INTFA_ERR_MISALIGNED;
    uint8_t *w = static_cast<uint8_t *>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t bytes = static_cast<size_t>(B) * H * L * d * 2;
    int rc = cuda_status(cudaMemcpyAsync(w + lo.hq, Q_f16_host, bytes, cudaMemcpyHostToDevice, s));
    if (!rc) rc = cuda_status(cudaMemcpyAsync(w + lo.hk, K_f16_host, bytes, cudaMemcpyHostToDevice, s));
    if (!rc) rc = cuda_status(cudaMemcpyAsync(w + lo.hv, V_f16_host, bytes, cudaMemcpyHostToDevice, s));
    if (!rc) rc = intfa_forward(w + lo.hq, w + lo.hk, w + lo.hv, B, H, L, d, causal, w + lo.ho,
                                workspace, lo.end, stream);
    if (!rc) rc = cuda_status(cudaMemcpyAsync(O_f16_host, w + lo.ho, bytes, cudaMemcpyDeviceToHost, s));
    return rc;
}
