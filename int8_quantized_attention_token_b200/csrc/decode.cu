// decode.cu -- INT8 attention for one query per head against a key / value
// cache (decode), sm_100a.
//
// Method: the online form of the fused kernel (INT-FlashAttention abstract;
// IntAttention eqs. 3-6, section 3.2, eq. 5) for a single query row: q is
// quantised per token (s_q = max|q| / 127), the cache holds K_hat with one
// scale per key and V_hat with one scale per head; per 128-key block
//   t_j = (q_hat . k_hat_j) s_q s_K[j] log2(e) / sqrt(d),  m_new = max(m, max_j t_j)
//   P_hat_j = RNE(127 2^(t_j - m_new)),  acc = 2^(m - m_new) acc + sum_j P_hat_j v_hat_j
//   l = 2^(m - m_new) l + sum_j 2^(t_j - m_new)
// with the keys cut into ranges of split_len keys that run these steps on
// their own (split-KV), merged by a second kernel:
//   M = max_s m_s,  O = s_V sum_s 2^(m_s - M) acc_s / (127 sum_s 2^(m_s - M) l_s).
//
// B200 design.  One query row is a matrix-vector product per head: a
// 128-row tensor-core MMA would waste 127 of its rows, and the path moves
// 2 d + 4 bytes of cache per key for 4 d operations, so it is bound by HBM.
// Kernel 1: one 128-thread CTA per (key range, head); the range's 128-key
// K_hat and V_hat blocks stream through a 3-stage shared-memory ring by bulk
// copies (the copy engine, one elected thread, mbarrier completion), two CTAs
// per SM.  Q K^T: D / 16 lanes per key, 16 bytes each, dp4a against the
// query's codes held in registers, a shuffle reduction; softmax one lane per
// key with warp / CTA reductions; P V: each thread owns 4 channels of the row
// and a quarter (D = 128) of the block's keys, one dp4a per channel and key.
// Kernel 2: the merge.  All waits are bounded.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"
#include "quant_math.cuh"

namespace intfa {

__device__ uint32_t g_status_decode;  // 0 = fine; else 0x300 | wait site of the first timeout

namespace {

constexpr int kThreads = 128;
constexpr int kBlk = 128;        // keys per block
constexpr int kStages = 3;
constexpr long long kWaitCycles = 1ll << 32;
constexpr uint32_t kSleepNs = 1000000;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: fl(y + kMagic) has RNE(y) in its low bits

template <int D>
struct alignas(128) DecSmem {
    int8_t k[kStages][kBlk * D];
    int8_t v[kStages][kBlk * D];
    uint64_t full[kStages];
    uint32_t qw[D / 4];          // the query's codes, four per word
    float sq;                    // its scale
    float red[2][4];             // per-warp partial max / sum
    uint8_t pcode[2][kBlk];      // P codes of the current block (two blocks in flight)
    float part[kThreads / (D / 4)][D];   // per key group accumulators, for the final sum
};

__device__ __forceinline__ bool wait_full(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity, kSleepNs)) {
        if (clock64() - t0 > kWaitCycles) {
            atomicCAS(&g_status_decode, 0u, 0x301u);
            return false;
        }
    }
    return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    decode_partial_kernel(const __half *__restrict__ q, const int8_t *__restrict__ Kq,
                          const float *__restrict__ sK, const int8_t *__restrict__ Vq, int L, int split_len,
                          float *__restrict__ ws) {
    constexpr int LPK = D / 16;          // lanes per key in Q K^T (16 bytes each)
    constexpr int KPI = 32 / LPK;        // keys per warp per step
    constexpr int NW = D / 4;            // channel words of a row
    constexpr int KG = kThreads / NW;    // key groups in P V
    extern __shared__ __align__(128) uint8_t smem_raw[];
    DecSmem<D> &sm = *reinterpret_cast<DecSmem<D> *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y, split = blockIdx.x;
    const int j_begin = split * split_len;
    const int j_end = min(L, j_begin + split_len);
    const int nblk = j_begin < L ? (j_end - j_begin + kBlk - 1) / kBlk : 0;
    float *out = ws + (static_cast<int64_t>(bh) * gridDim.x + split) * (D + 2);
    if (nblk == 0) {   // an empty range (more ranges than the cache needs)
        if (tid == 0) {
            out[0] = -INFINITY;
            out[1] = 0.0f;
        }
        for (int c = tid; c < D; c += kThreads) out[2 + c] = 0.0f;
        return;
    }
    const int8_t *Kh = Kq + static_cast<int64_t>(bh) * L * D;
    const int8_t *Vh = Vq + static_cast<int64_t>(bh) * L * D;
    const float *sKh = sK + static_cast<int64_t>(bh) * L;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[s], 1);
        fence_mbar_init();
    }
    // the query row, quantised per token (the standalone quantiser's arithmetic)
    if (warp == 0) {
        constexpr int G = D / 8;   // lanes of 8 elements
        float f[8];
        float amax = 0.0f;
        if (lane < G) {
            qmath::unpack8(reinterpret_cast<const uint4 *>(q + static_cast<int64_t>(bh) * D)[lane], f);
            amax = qmath::absmax8(f);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        const float s = qmath::div127(amax);
        if (lane < G) {
            const uint2 w = qmath::codes8(f, s, qmath::rcp_or_zero(s));
            sm.qw[2 * lane] = w.x;
            sm.qw[2 * lane + 1] = w.y;
        }
        if (lane == 0) sm.sq = s;
    }
    __syncthreads();
    auto issue = [&](int b) {
        const int st = b % kStages;
        const int j0 = j_begin + b * kBlk;
        const uint32_t bytes = static_cast<uint32_t>(min(kBlk, j_end - j0) * D);
        mbar_arrive_expect_tx(&sm.full[st], 2 * bytes);
        bulk_g2s(sm.k[st], Kh + static_cast<int64_t>(j0) * D, bytes, &sm.full[st]);
        bulk_g2s(sm.v[st], Vh + static_cast<int64_t>(j0) * D, bytes, &sm.full[st]);
    };
    if (tid == 0)
        for (int b = 0; b < kStages && b < nblk; ++b) issue(b);

    const int seg = lane % LPK;
    const uint4 q4 = make_uint4(sm.qw[4 * seg], sm.qw[4 * seg + 1], sm.qw[4 * seg + 2], sm.qw[4 * seg + 3]);
    const float c = sm.sq * (kLog2e / sqrtf(static_cast<float>(D)));
    const int cw = tid % NW, kg = tid / NW;
    float m = -INFINITY, l = 0.0f;
    float facc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    bool ok = true;
    for (int b = 0; b < nblk; ++b) {
        const int st = b % kStages;
        const int j0 = j_begin + b * kBlk;
        const int n = min(kBlk, j_end - j0);
        const int key = 32 * warp + lane;   // this lane's key in the softmax
        const float skj = key < n ? __ldg(sKh + j0 + key) : 0.0f;
        if (!wait_full(&sm.full[st], (b / kStages) & 1)) ok = false;
        if (!__syncthreads_and(ok)) break;
        // -- Q K^T: warp w, keys 32 w .. 32 w + 31, KPI keys per step
        int sdot = 0;
#pragma unroll
        for (int it = 0; it < LPK; ++it) {
            const int kk = 32 * warp + it * KPI + lane / LPK;
            const uint4 kv = *reinterpret_cast<const uint4 *>(sm.k[st] + kk * D + 16 * seg);
            int a = __dp4a(static_cast<int>(kv.x), static_cast<int>(q4.x), 0);
            a = __dp4a(static_cast<int>(kv.y), static_cast<int>(q4.y), a);
            a = __dp4a(static_cast<int>(kv.z), static_cast<int>(q4.z), a);
            a = __dp4a(static_cast<int>(kv.w), static_cast<int>(q4.w), a);
#pragma unroll
            for (int o = LPK / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
            // lane j takes key j's sum from step j / KPI, lane (j mod KPI) LPK
            const int got = __shfl_sync(0xFFFFFFFFu, a, (lane % KPI) * LPK);
            if (lane / KPI == it) sdot = got;
        }
        const float t = key < n ? static_cast<float>(sdot) * skj * c : -INFINITY;
        // -- block max, running max
        float bm = t;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xFFFFFFFFu, bm, o));
        if (lane == 0) sm.red[0][warp] = bm;
        __syncthreads();
        const float m_new = fmaxf(m, fmaxf(fmaxf(sm.red[0][0], sm.red[0][1]), fmaxf(sm.red[0][2], sm.red[0][3])));
        const float alpha = exp2f(m - m_new);   // 0 for the first block (m = -inf)
        // -- p, P codes, row sum
        const float p = exp2f(t - m_new);
        sm.pcode[b & 1][key] = static_cast<uint8_t>(__float_as_uint(fmaf(p, 127.0f, kMagic)) & 0xFFu);
        float ps = p;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, o);
        if (lane == 0) sm.red[1][warp] = ps;
        __syncthreads();
        l = alpha * l + ((sm.red[1][0] + sm.red[1][1]) + (sm.red[1][2] + sm.red[1][3]));
        // -- P V: channels 4 cw .. 4 cw + 3, keys kg, kg + KG, ...
        int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll 4
        for (int kk = kg; kk < kBlk; kk += KG) {
            const int pc = sm.pcode[b & 1][kk];   // 0 past the end of the range
            const int vw = *reinterpret_cast<const int *>(sm.v[st] + kk * D + 4 * cw);
            a0 = __dp4a(vw, pc, a0);
            a1 = __dp4a(vw, pc << 8, a1);
            a2 = __dp4a(vw, pc << 16, a2);
            a3 = __dp4a(vw, pc << 24, a3);
        }
        facc[0] = fmaf(alpha, facc[0], static_cast<float>(a0));
        facc[1] = fmaf(alpha, facc[1], static_cast<float>(a1));
        facc[2] = fmaf(alpha, facc[2], static_cast<float>(a2));
        facc[3] = fmaf(alpha, facc[3], static_cast<float>(a3));
        m = m_new;
        __syncthreads();   // stage st and the P codes of block b are no longer read
        if (tid == 0 && b + kStages < nblk) issue(b + kStages);
    }
    if (!ok) {   // a copy never arrived: report an empty range
        if (tid == 0) {
            out[0] = -INFINITY;
            out[1] = 0.0f;
        }
        for (int cc = tid; cc < D; cc += kThreads) out[2 + cc] = 0.0f;
        return;
    }
    // the key groups' partial sums -> the range's accumulator
#pragma unroll
    for (int e = 0; e < 4; ++e) sm.part[kg][4 * cw + e] = facc[e];
    __syncthreads();
    for (int cc = tid; cc < D; cc += kThreads) {
        float s = 0.0f;
#pragma unroll
        for (int g = 0; g < KG; ++g) s += sm.part[g][cc];
        out[2 + cc] = s;
    }
    if (tid == 0) {
        out[0] = m;
        out[1] = l;
    }
}

// O = s_V sum_s 2^(m_s - M) acc_s / (127 sum_s 2^(m_s - M) l_s), one CTA per head.
template <int D>
__global__ void __launch_bounds__(D)
    decode_combine_kernel(const float *__restrict__ ws, int nsplit, const float *__restrict__ sV,
                          __half *__restrict__ O) {
    const int bh = blockIdx.x, cc = threadIdx.x;
    const float *w = ws + static_cast<int64_t>(bh) * nsplit * (D + 2);
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) M = fmaxf(M, w[s * (D + 2)]);
    float num = 0.0f, den = 0.0f;
    for (int s = 0; s < nsplit; ++s) {
        const float ms = w[s * (D + 2)];
        const float f = ms == -INFINITY ? 0.0f : exp2f(ms - M);
        den = fmaf(f, w[s * (D + 2) + 1], den);
        num = fmaf(f, w[s * (D + 2) + 2 + cc], num);
    }
    O[static_cast<int64_t>(bh) * D + cc] = __float2half_rn(__ldg(sV + bh) * num / (127.0f * den));
}

template <int D>
int launch_decode(const void *q, const int8_t *Kq, const float *sK, const int8_t *Vq, const float *sV, int BH,
                  int L, int splits, void *O, float *ws, cudaStream_t stream) {
    const int nblk = (L + kBlk - 1) / kBlk;
    const int split_len = ((nblk + splits - 1) / splits) * kBlk;
    const size_t smem = sizeof(DecSmem<D>);
    int rc = cuda_status(cudaFuncSetAttribute(decode_partial_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(smem)));
    if (rc) return rc;
    decode_partial_kernel<D><<<dim3(static_cast<unsigned>(splits), static_cast<unsigned>(BH)), kThreads, smem,
                               stream>>>(static_cast<const __half *>(q), Kq, sK, Vq, L, split_len, ws);
    rc = cuda_status(cudaGetLastError());
    if (rc) return rc;
    decode_combine_kernel<D><<<static_cast<unsigned>(BH), D, 0, stream>>>(ws, splits, sV, static_cast<__half *>(O));
    return cuda_status(cudaGetLastError());
}

}  // namespace

int read_decode_status(int clear, uint32_t *word) {
    uint32_t w = 0;
    int rc = cuda_status(cudaMemcpyFromSymbol(&w, g_status_decode, sizeof(w)));
    if (rc) return rc;
    if (clear) {
        const uint32_t z = 0;
        rc = cuda_status(cudaMemcpyToSymbol(g_status_decode, &z, sizeof(z)));
        if (rc) return rc;
    }
    *word = w;
    return INTFA_OK;
}

}  // namespace intfa

// ------------------------------------------------------------------ C ABI ---

extern "C" size_t intfa_decode_workspace_size(int B, int H, int d, int splits) {
    if (B <= 0 || H <= 0 || splits <= 0 || (d != 64 && d != 128)) return 0;
    return static_cast<size_t>(B) * H * splits * (d + 2) * sizeof(float);
}

extern "C" int intfa_decode_fwd(const void *q_f16, const int8_t *K_q, const float *s_K, const int8_t *V_q,
                                const float *s_V, int B, int H, int L, int d, int splits, void *O_f16,
                                void *workspace, size_t workspace_bytes, void *stream) {
    using namespace intfa;
    if (B <= 0 || H <= 0 || L <= 0 || splits <= 0 || splits > 65535) return INTFA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return INTFA_ERR_UNSUPPORTED;
    const int64_t bh = static_cast<int64_t>(B) * H;
    if (bh > 65535 || L > (1 << 24)) return INTFA_ERR_UNSUPPORTED;
    if (!q_f16 || !K_q || !s_K || !V_q || !s_V || !O_f16 || !workspace) return INTFA_ERR_INVALID_ARG;
    if (workspace_bytes < intfa_decode_workspace_size(B, H, d, splits)) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(q_f16) || !aligned16(K_q) || !aligned16(V_q) || !aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(s_K) & 3u) || (reinterpret_cast<uintptr_t>(s_V) & 3u) ||
        (reinterpret_cast<uintptr_t>(O_f16) & 1u))
        return INTFA_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *ws = static_cast<float *>(workspace);
    if (d == 128) return launch_decode<128>(q_f16, K_q, s_K, V_q, s_V, static_cast<int>(bh), L, splits, O_f16, ws, s);
    return launch_decode<64>(q_f16, K_q, s_K, V_q, s_V, static_cast<int>(bh), L, splits, O_f16, ws, s);
}
