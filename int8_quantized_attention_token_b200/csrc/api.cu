// api.cu -- the whole-path entry points of libintfa (quantise Q/K per token,
// V per head, then the fused attention; and the same from host buffers) and
// the status strings.  See include/intfa.h for the contract of each call.
#include <mutex>

#include "internal.h"

namespace {

struct Layout {
    size_t q, k, v, sq, sk, sv, ws, end;        // device workspace of intfa_forward
    size_t hq, hk, hv, ho, host_end;           // + fp16 staging for intfa_forward_host
};

bool make_layout(int B, int H, int L, int d, Layout *lo) {
    if (B <= 0 || H <= 0 || L <= 0 || (d != 64 && d != 128)) return false;
    const size_t bh = static_cast<size_t>(B) * H;
    if (bh > (1u << 24) || L > 131072) return false;
    if (bh * ((static_cast<size_t>(L) + 127) / 128) > 0x7FFFFFFFu) return false;   // tile count fits an int
    const size_t n = bh * static_cast<size_t>(L);              // token rows
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = intfa::round_up(off + bytes, 256);
        return at;
    };
    lo->q = take(n * d);
    lo->k = take(n * d);
    lo->v = take(n * d);                                       // V_hat, untransposed
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
    offsets[2] = lo.v;
    offsets[3] = lo.sq;
    offsets[4] = lo.sk;
    offsets[5] = lo.sv;
    return INTFA_OK;
}

namespace {

// Streams and events of one device: the pipelined host path's copy streams,
// and intfa_forward's side stream.  Made on the first call on that device and
// kept for the life of the process (no allocation of device memory; nothing
// is created on later calls).
struct HostPipe {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, in = nullptr, out = nullptr, done = nullptr;
    cudaStream_t side = nullptr;                   // intfa_forward: V's quantiser beside Q's and K's
    cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxDevices = 64;
std::mutex g_pipe_mu;             // guards g_pipes and keeps each call's enqueue sequence whole
HostPipe g_pipes[kMaxDevices];

int get_pipe(HostPipe **out) {
    int dev = 0;
    int rc = intfa::cuda_status(cudaGetDevice(&dev));
    if (rc) return rc;
    if (dev < 0 || dev >= kMaxDevices) return INTFA_ERR_UNSUPPORTED;
    HostPipe &p = g_pipes[dev];
    if (!p.done) {
        HostPipe n;
        rc = intfa::cuda_status(cudaStreamCreateWithFlags(&n.h2d, cudaStreamNonBlocking));
        if (!rc) rc = intfa::cuda_status(cudaStreamCreateWithFlags(&n.d2h, cudaStreamNonBlocking));
        if (!rc) rc = intfa::cuda_status(cudaEventCreateWithFlags(&n.start, cudaEventDisableTiming));
        if (!rc) rc = intfa::cuda_status(cudaEventCreateWithFlags(&n.in, cudaEventDisableTiming));
        if (!rc) rc = intfa::cuda_status(cudaEventCreateWithFlags(&n.out, cudaEventDisableTiming));
        if (!rc) rc = intfa::cuda_status(cudaEventCreateWithFlags(&n.done, cudaEventDisableTiming));
        if (!rc) rc = intfa::cuda_status(cudaStreamCreateWithFlags(&n.side, cudaStreamNonBlocking));
        if (!rc) rc = intfa::cuda_status(cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming));
        if (!rc) rc = intfa::cuda_status(cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming));
        if (rc) {
            for (cudaStream_t t : {n.h2d, n.d2h, n.side})
                if (t) cudaStreamDestroy(t);
            for (cudaEvent_t e : {n.start, n.in, n.out, n.done, n.fork, n.join})
                if (e) cudaEventDestroy(e);
            return rc;
        }
        p = n;
    }
    *out = &p;
    return INTFA_OK;
}

}  // namespace

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
    int8_t *v = reinterpret_cast<int8_t *>(w + lo.v);
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
    std::lock_guard<std::mutex> lock(g_pipe_mu);   // keeps this call's fork / join whole
    HostPipe *pp = nullptr;
    int rc = get_pipe(&pp);
    if (rc) return rc;
    // V's quantiser (V_hat stays in V's layout: the attention reads its tiles
    // N-major) runs on the library's side stream while Q's and K's run on the
    // caller's; the three are HBM-bound and fill each other's gaps (measured
    // on B4 H32 L4096 d128: 131 -> 115 us for the three).  The caller's stream
    // waits for the side stream before the attention, whatever happened.
    rc = cuda_status(cudaEventRecord(pp->fork, s));
    if (!rc) rc = cuda_status(cudaStreamWaitEvent(pp->side, pp->fork, 0));
    if (!rc) rc = launch_quantize_per_tensor(V_f16, bh, L, d, 0, v, sv, w + lo.ws, pp->side);
    if (!rc) rc = launch_quantize_per_token(Q_f16, rows, d, q, sq, s);
    if (!rc) rc = launch_quantize_per_token(K_f16, rows, d, k, sk, s);
    int rc2 = cuda_status(cudaEventRecord(pp->join, pp->side));
    if (!rc2) rc2 = cuda_status(cudaStreamWaitEvent(s, pp->join, 0));
    if (!rc && !rc2) rc = launch_attention_fwd_vrows(q, k, v, sq, sk, sv, B, H, L, d, causal, O_f16, s);
    return rc ? rc : rc2;
}

namespace {

// Heads in the next chunk of the host pipeline, rem heads left: half of them
// (large chunks first keep the launches efficient, small ones last keep the
// tail after the final input copy short), and at least 4 MiB of fp16 per
// tensor per copy so that each copy runs at full link speed.  (Measured on
// B4 H32 L4096 d128 causal, ms per call: halving 8.01; equal chunks, 4: 8.47,
// 6: 8.26, 8: 8.35, 12: 8.35, 16: 8.58-8.72, 32: 8.62, 64: 9.22.)
int64_t next_chunk_heads(int64_t rem, int64_t head_bytes) {
    const int64_t by_size = ((int64_t{4} << 20) + head_bytes - 1) / head_bytes;
    const int64_t half = (rem + 1) / 2;
    const int64_t nh = half > by_size ? half : by_size;
    return nh < rem ? nh : rem;
}

}  // namespace

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
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    if (!Q_f16_host || !K_f16_host || !V_f16_host || !O_f16_host) return INTFA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < lo.host_end) return INTFA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return INTFA_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lock(g_pipe_mu);
    HostPipe *pp = nullptr;
    int rc = get_pipe(&pp);
    if (rc) return rc;
    const HostPipe &pipe = *pp;
    uint8_t *w = static_cast<uint8_t *>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t bh = static_cast<int64_t>(B) * H;
    const size_t head_bytes = static_cast<size_t>(L) * d * 2;   // fp16 of one head
    // Heads are independent: chunk c's host-to-device copies (stream h2d),
    // its quantisation and attention (the caller's stream) and its output copy
    // (stream d2h) overlap with the neighbouring chunks' copies in the other
    // direction.  Every chunk owns its own slice of the staging buffers, so
    // nothing is overwritten while still in use.
    rc = cuda_status(cudaEventRecord(pipe.start, s));   // work already queued on the caller's stream
    if (!rc) rc = cuda_status(cudaStreamWaitEvent(pipe.h2d, pipe.start, 0));
    if (!rc) rc = cuda_status(cudaStreamWaitEvent(pipe.d2h, pipe.start, 0));
    for (int64_t h0 = 0, nh = 0; !rc && h0 < bh; h0 += nh) {
        nh = next_chunk_heads(bh - h0, static_cast<int64_t>(head_bytes));
        const size_t off = static_cast<size_t>(h0) * head_bytes, bytes = static_cast<size_t>(nh) * head_bytes;
        rc = cuda_status(cudaMemcpyAsync(w + lo.hq + off, static_cast<const uint8_t *>(Q_f16_host) + off, bytes,
                                         cudaMemcpyHostToDevice, pipe.h2d));
        if (!rc) rc = cuda_status(cudaMemcpyAsync(w + lo.hk + off, static_cast<const uint8_t *>(K_f16_host) + off,
                                                  bytes, cudaMemcpyHostToDevice, pipe.h2d));
        if (!rc) rc = cuda_status(cudaMemcpyAsync(w + lo.hv + off, static_cast<const uint8_t *>(V_f16_host) + off,
                                                  bytes, cudaMemcpyHostToDevice, pipe.h2d));
        if (!rc) rc = cuda_status(cudaEventRecord(pipe.in, pipe.h2d));
        if (!rc) rc = cuda_status(cudaStreamWaitEvent(s, pipe.in, 0));
        const int64_t rows = nh * L, r0 = h0 * L;
        int8_t *q = reinterpret_cast<int8_t *>(w + lo.q) + r0 * d;
        int8_t *k = reinterpret_cast<int8_t *>(w + lo.k) + r0 * d;
        int8_t *v = reinterpret_cast<int8_t *>(w + lo.v) + r0 * d;
        float *sq = reinterpret_cast<float *>(w + lo.sq) + r0;
        float *sk = reinterpret_cast<float *>(w + lo.sk) + r0;
        float *sv = reinterpret_cast<float *>(w + lo.sv) + h0;
        if (!rc) rc = launch_quantize_per_token(w + lo.hq + off, rows, d, q, sq, s);
        if (!rc) rc = launch_quantize_per_token(w + lo.hk + off, rows, d, k, sk, s);
        if (!rc) rc = launch_quantize_per_tensor(w + lo.hv + off, nh, L, d, 0, v, sv, w + lo.ws, s);
        if (!rc) rc = launch_attention_fwd_vrows(q, k, v, sq, sk, sv, 1, static_cast<int>(nh), L, d, causal,
                                                 w + lo.ho + off, s);
        if (!rc) rc = cuda_status(cudaEventRecord(pipe.out, s));
        if (!rc) rc = cuda_status(cudaStreamWaitEvent(pipe.d2h, pipe.out, 0));
        if (!rc) rc = cuda_status(cudaMemcpyAsync(static_cast<uint8_t *>(O_f16_host) + off, w + lo.ho + off, bytes,
                                                  cudaMemcpyDeviceToHost, pipe.d2h));
    }
    // Whatever happened above, the caller's stream ends behind both copy
    // streams, so synchronising it covers every copy this call queued.
    int rc2 = cuda_status(cudaEventRecord(pipe.in, pipe.h2d));
    if (!rc2) rc2 = cuda_status(cudaStreamWaitEvent(pipe.d2h, pipe.in, 0));
    if (!rc2) rc2 = cuda_status(cudaEventRecord(pipe.done, pipe.d2h));
    if (!rc2) rc2 = cuda_status(cudaStreamWaitEvent(s, pipe.done, 0));
    return rc ? rc : rc2;
}
