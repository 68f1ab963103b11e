// index_attention.cu -- IndexSoftmax attention forward pass for sm_100a.
//
// Method (IntAttention: A Fully Integer Attention Pipeline for Efficient Edge
// Inference, section 3.1 eqs. 7-10 and section 3.2; eq. 5 for the value
// path), with per-tensor Q / K / V scales (section 3.3's default):
//   A_hat  = Q_hat K_hat^T                          INT8 x INT8 -> INT32
//   m_i    = max over visible keys j of A_hat[i, j]          (pass A, eq. 7)
//   D'_ij  = min(m_i - A_hat[i, j], c_int),  c_int = rint(c sqrt(d) / (s_Q s_K))
//   idx    = floor(D' (2^b - 1) / c_int)                      (eqs. 8-10)
//   E_ij   = LUT[idx],  LUT[k] = rint(255 exp(-c k / (2^b - 1)))   (UINT8)
//   acc_i  = sum_j E_ij V_hat_j                     UINT8 x INT8 -> INT32
//   l_i    = sum_j E_ij                             (integer row sum)
//   O_i    = s_V acc_i / l_i                        -> fp16
// The row max is taken over the whole row before any table lookup (the
// pages' two-pass form), so the integer accumulators need no rescaling: the
// P V products of all key blocks accumulate in TMEM.
//
// B200 design: one CTA per (128-query tile, head), 10 warps:
//   warps 0-7  two threads per query row: warp w reads TMEM lane quadrant
//              w mod 4 and key half w / 4 (64 of each block's 128 keys).
//              Pass A: the half's row max; the two halves meet once, through
//              shared memory, after the last block.  Pass B: distances,
//              table lookups, P codes of the half's keys and its integer row
//              sum; the halves add their sums once at the end and each
//              writes half of the output row.
//   warp 8     TMA producer: the Q_hat tile, then for each of the 2 nb steps
//              (nb key blocks, twice) the K_hat tile and, in pass B, the
//              V_hat^T tile, through a 2-stage ring.
//   warp 9     MMA issuer (one lane), TMEM owner: Q K^T of every step into
//              the S buffer (first set to a float bias by an fp16 MMA
//              so that S reads back as fp32 exactly), and in pass B the P V
//              products, accumulated in an int32 TMEM block.
// Two CTAs share an SM (256 TMEM columns, 96 registers per thread and ~84 KB
// of shared memory each): one CTA's row warps work while the other's MMAs
// run, in place of a second S buffer within the CTA.
// Every wait is bounded (clock-based); a timeout records a status word,
// raises a CTA-wide abort flag, drains in-flight copies and MMAs, frees TMEM
// and returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"
#include "tma_host.h"

namespace intfa {

__device__ uint32_t g_status_index;  // 0 = fine; else 0x200 | wait site of the first timeout

namespace {

constexpr int BM = 128;                 // query rows per CTA
constexpr int BN = 128;                 // keys per block
constexpr int NS = 2;                   // K / V ring depth
constexpr int SB = 1;                   // TMEM S buffers (two CTAs per SM overlap each other's steps)
constexpr int kMinBlocks = 2;           // CTAs per SM: TMEM, registers and shared memory sized for two
constexpr int kParts = 2;          // row warps per TMEM lane quadrant (key parts of a block)
static_assert(kParts == 1 || kParts == 2 || kParts == 4, "a block's 4 chunks split evenly");
constexpr int kRowWarps = 4 * kParts;
constexpr int kChunks = 4 / kParts;     // 32-key chunks of a block per row warp
constexpr int kThreads = 32 * (kRowWarps + 2);
constexpr int kProducerWarp = kRowWarps;
constexpr int kMmaWarp = kRowWarps + 1;
constexpr int kRowBarrier = 1;          // named barrier of the row warps
constexpr int kTmemCols = 256;          // the S buffer (128 columns) + the P V accumulator (<= 128)
static_assert(SB * BN + 128 <= kTmemCols, "TMEM columns");
constexpr long long kWaitCycles = 1ll << 32;  // ~2 s at B200 clocks
constexpr uint32_t kSleepNs = 1000000;
// Accumulator bias: 1.5 * 2^23 as fp32 has the bit pattern 0x4B400000; an
// INT8 MMA adding the int32 S to it leaves the bit pattern of the float
// 1.5 * 2^23 + S (|S| <= 127^2 * 128 < 2^22).  The fp16 bias MMA writes that
// float as 16 exact products 1024 * 768.
constexpr float kBias = 12582912.0f;
constexpr uint16_t kBiasA = 0x6400;     // fp16 1024
constexpr uint16_t kBiasB = 0x6200;     // fp16 768

template <int D>
struct alignas(1024) IdxSmem {
    uint8_t q[BM * D];          // Q_hat tile, K-major, TMA-swizzled
    uint8_t k[NS][BN * D];      // K_hat tiles
    uint8_t v[NS][D * BN];      // V_hat^T tiles (row = channel, 128 keys)
    uint8_t lut[256];           // the UINT8 exponential table (2^b entries used)
    uint16_t bias_ab[2][192];   // fp16 operands of the bias MMA
    uint64_t q_full;
    uint64_t full[NS], empty[NS];   // ring stage loaded / released
    uint64_t s_full[SB];        // Q K^T of the step in buffer b done
    uint64_t s_read[SB];        // pass A: the row warps have read buffer b
    uint64_t p_full[SB];        // pass B: P codes of the step in buffer b written
    uint64_t pv_done[SB];       // pass B: P V of the step in buffer b done
    uint64_t acc_full;          // all P V products of the tile done
    uint64_t mma_drain;
    float half_max[kParts][BM];      // each key part's row max (biased float)
    uint32_t half_sum[kParts][BM];   // each key part's integer row sum
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
constexpr size_t idx_smem_bytes() { return sizeof(IdxSmem<D>) + 1024; }
static_assert(idx_smem_bytes<128>() <= 227 * 1024 && idx_smem_bytes<64>() <= 227 * 1024,
              "shared memory above the per-block limit");

__device__ __forceinline__ uint8_t *smem_base_1024() {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t off = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    return smem_raw + off;
}

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         uint32_t site) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity, kSleepNs)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitCycles) {
            *abort_flag = 1;
            atomicCAS(&g_status_index, 0u, 0x200u | site);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          uint32_t site) {
    const bool ok = wait_bar(bar, parity, abort_flag, site);
    return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity, kSleepNs)) {
        if (clock64() - t0 > kWaitCycles) {
            atomicCAS(&g_status_index, 0u, 0x2FFu);
            return;
        }
    }
}

// One byte of shared memory at a 32-bit shared-window address.
__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// The row warps (warps 0-7) meet: every row warp reaches each call exactly
// once, whatever happened to its waits before.
__device__ __forceinline__ void row_barrier() {
    asm volatile("bar.sync %0, %1;" ::"n"(kRowBarrier), "n"(32 * kRowWarps) : "memory");
}

// c_int of eq. 8 in fp64: rint((c sqrt(d)) / (s_Q s_K)), at least 1 (and at
// most 4e18); a zero scale gives 1 (all logits are then 0).
__device__ __forceinline__ long long clip_threshold(double c, int d, float sQ, float sK) {
    const double den = __dmul_rn(static_cast<double>(sQ), static_cast<double>(sK));
    if (!(den > 0.0)) return 1;
    const double v = rint(__ddiv_rn(__dmul_rn(c, sqrt(static_cast<double>(d))), den));
    if (v < 1.0) return 1;
    if (v > 4.0e18) return 4000000000000000000ll;
    return static_cast<long long>(v);
}

// Pass A: keys at or past lim get 0, below every biased logit (> 2^22).
__device__ __forceinline__ void mask_zero(uint32_t (&w)[32], int key0, int lim) {
#pragma unroll
    for (int e = 0; e < 32; ++e)
        if (key0 + e >= lim) w[e] = 0u;
}

__device__ __forceinline__ void max_chunk(const uint32_t (&w)[32], float (&mx)[4]) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
        mx[q & 3] = fmax3(mx[q & 3], fmax3(__uint_as_float(w[4 * q]), __uint_as_float(w[4 * q + 1]),
                                           __uint_as_float(w[4 * q + 2])),
                          __uint_as_float(w[4 * q + 3]));
}

// Pass B for one 32-key chunk: E = LUT[idx] (0 for masked keys), packed four
// per word in key order, and the integer row sum.  kFast: idx =
// floor(D' q) with q = (2^b - 1) / c_int rounded up, evaluated as the
// round-down fma D' q + 2^23 (exact for c_int <= 2^(23 - b), see the launch
// comment); otherwise the integer quotient.
template <bool kFast, bool kMask>
__device__ __forceinline__ void lookup_chunk(const uint32_t (&w)[32], float mbf, float cf, float q,
                                             unsigned long long cint, uint32_t nm1,
                                             const uint8_t *lut, uint32_t lut_biased, int key0, int lim,
                                             uint32_t &l, uint32_t (&pk)[8]) {
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        uint32_t e[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const bool masked = kMask && key0 + 4 * g + t >= lim;
            if constexpr (kFast) {
                // a masked key looks up D' = 0 (its value is zeroed below);
                // a visible one has 0 <= D' <= c_int, so D' q + 2^23 rounded
                // down is 0x4B000000 + idx with idx <= 2^b - 1, and adding its
                // bits to the table's shared address minus 0x4B000000 gives
                // the entry's address in one integer add
                const float sv = masked ? mbf : __uint_as_float(w[4 * g + t]);
                const float dl = fminf(mbf - sv, cf);   // exact: both are integers + 1.5 * 2^23
                e[t] = lds_u8(lut_biased + __float_as_uint(__fmaf_rd(dl, q, 8388608.0f)));
            } else {
                const float dl = fminf(mbf - __uint_as_float(w[4 * g + t]), cf);
                uint32_t idx = static_cast<uint32_t>((static_cast<unsigned long long>(dl) * nm1) / cint);
                idx = min(idx, nm1);
                e[t] = lut[idx];
            }
            if (masked) e[t] = 0u;
        }
        pk[g] = prmt(prmt(e[0], e[1], 0x0040u), prmt(e[2], e[3], 0x0040u), 0x5410u);
        l = __dp4a(pk[g], 0x01010101u, l);
    }
}

template <bool kFast, int NCH>
__device__ __forceinline__ void lookup_block(uint32_t (&w)[NCH][32], float mbf, float cf, float q,
                                             unsigned long long cint, uint32_t nm1, const uint8_t *lut,
                                             bool need_mask, int key0, int lim, uint32_t &l,
                                             uint32_t ts) {
    const uint32_t lut_biased = smem_u32(lut) - 0x4B000000u;   // wraps; the add in lookup_chunk wraps back
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
        uint32_t pk[8];
        if (need_mask)
            lookup_chunk<kFast, true>(w[ch], mbf, cf, q, cint, nm1, lut, lut_biased, key0 + 32 * ch, lim, l, pk);
        else
            lookup_chunk<kFast, false>(w[ch], mbf, cf, q, cint, nm1, lut, lut_biased, key0 + 32 * ch, lim, l, pk);
        tmem_st8(ts + 32 * ch, pk);   // codes of keys 32 ch .. 32 ch + 31: the A operand of P V step ch
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
    attn_index_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const float *__restrict__ sQ,
                      const float *__restrict__ sK, const float *__restrict__ sV,
                      __half *__restrict__ O, int L, int causal, double c, int bits,
                      int32_t *__restrict__ m_out, int32_t *__restrict__ l_out) {
    IdxSmem<D> &sm = *reinterpret_cast<IdxSmem<D> *>(smem_base_1024());
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = (L + BM - 1) / BM;
    const int qt = ntiles - 1 - static_cast<int>(blockIdx.x);   // heaviest causal tiles first
    const int bh = blockIdx.y;
    const int q0 = qt * BM;
    const int nb = causal ? qt + 1 : (L + BN - 1) / BN;
    const int T = 2 * nb;                                        // steps: pass A, then pass B
    const uint32_t nm1 = (1u << bits) - 1u;
    volatile int *abort_flag = &sm.abort_flag;

    if (tid == 0) {
        mbar_init(&sm.q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < SB; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.s_read[b], kParts * BM);   // every row warp reads its part
            mbar_init(&sm.p_full[b], kParts * BM);
            mbar_init(&sm.pv_done[b], 1);
        }
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.mma_drain, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    // the exponential table, in fp64 as (c k) / (2^b - 1), then 255 exp(-x), RNE
    for (uint32_t k = tid; k <= nm1; k += kThreads) {
        const double x = __ddiv_rn(__dmul_rn(c, static_cast<double>(k)), static_cast<double>(nm1));
        sm.lut[k] = static_cast<uint8_t>(rint(__dmul_rn(255.0, exp(-x))));
    }
    for (int e = tid; e < 2 * 192; e += kThreads) sm.bias_ab[e / 192][e % 192] = e < 192 ? kBiasA : kBiasB;
    fence_proxy_async_smem();   // the bias operands are read by the tensor core
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tS = sm.tmem_base;           // S buffer b at column 128 b
    const uint32_t tO = sm.tmem_base + SB * BN;  // int32 P V accumulator

    if (warp == kProducerWarp) {
        // ----------------------------------------------- TMA producer ---
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(&sm.q_full, BM * D);
            tma_load_3d(&tmQ, &sm.q_full, sm.q, 0, q0, bh);
            int s = 0;
            for (; s < T; ++s) {
                const int st = s % NS;
                if (s >= NS && !wait_bar(&sm.empty[st], ((s / NS) - 1) & 1, abort_flag, 7)) break;
                const bool pass_b = s >= nb;
                const int j = pass_b ? s - nb : s;
                mbar_arrive_expect_tx(&sm.full[st], BN * D + (pass_b ? D * BN : 0));
                tma_load_3d(&tmK, &sm.full[st], sm.k[st], 0, j * BN, bh);
                if (pass_b) tma_load_3d(&tmV, &sm.full[st], sm.v[st], j * BN, 0, bh);
            }
            // Drain: the Q tile and the last load into each stage have landed.
            drain_wait(&sm.q_full, 0);
            for (int st = 0; st < NS && st < s; ++st) {
                const int last = st + ((s - 1 - st) / NS) * NS;
                drain_wait(&sm.full[st], (last / NS) & 1);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer ---
        if (lane == 0) {
            constexpr uint32_t kSw = (D == 128) ? kSwizzle128B : kSwizzle64B;
            constexpr uint32_t kSbo = 8 * D;
            const uint32_t idesc_qk = make_idesc_i8(BM, BN);
            const uint32_t idesc_pv = make_idesc_u8s8(BM, D);
            const uint32_t idesc_bias = make_idesc_f16(BM, BN);
            // constant operands: overlapping core matrices are harmless (16-byte
            // strides keep every read inside the 384-byte arrays)
            const uint64_t bias_a = make_sdesc_noswz(smem_u32(sm.bias_ab[0]), 16, 16);
            const uint64_t bias_b = make_sdesc_noswz(smem_u32(sm.bias_ab[1]), 16, 16);
            const uint64_t qdesc = make_sdesc(smem_u32(sm.q), kSbo, kSw);
            uint32_t n_read[SB] = {}, n_pv[SB] = {}, n_p[SB] = {};
            bool ok = wait_bar(&sm.q_full, 0, abort_flag, 2);
            // Q K^T of step s into S buffer s mod 2, once the step two back has
            // released it (pass A: the row warps read it; pass B: its P V ran)
            auto issue_qk = [&](int s) -> bool {
                const int st = s % NS, b = s % SB;
                if (!wait_bar(&sm.full[st], (s / NS) & 1, abort_flag, 3)) return false;
                if (s >= SB) {
                    if (s - SB < nb) {
                        if (!wait_bar(&sm.s_read[b], n_read[b] & 1, abort_flag, 4)) return false;
                        ++n_read[b];
                    } else {
                        if (!wait_bar(&sm.pv_done[b], n_pv[b] & 1, abort_flag, 5)) return false;
                        ++n_pv[b];
                    }
                }
                tc_fence_after();
                const uint64_t kdesc = make_sdesc(smem_u32(sm.k[st]), kSbo, kSw);
                mma_f16_ss(tS + b * BN, bias_a, bias_b, idesc_bias, 0);
#pragma unroll
                for (int k = 0; k < D / 32; ++k)
                    mma_i8_ss(tS + b * BN, qdesc + 2 * k, kdesc + 2 * k, idesc_qk, 1);
                mma_commit(&sm.s_full[b]);
                if (s < nb) mma_commit(&sm.empty[st]);   // pass A: only the K tile was used
                return true;
            };
            for (int s0 = 0; ok && s0 < SB && s0 < T; ++s0) ok = issue_qk(s0);
            for (int s = 0; ok && s < T; ++s) {
                if (s >= nb) {
                    const int j = s - nb, b = s % SB, st = s % NS;
                    if (!wait_bar(&sm.p_full[b], n_p[b] & 1, abort_flag, 6)) break;
                    ++n_p[b];
                    tc_fence_after();
                    const uint64_t vdesc = make_sdesc(smem_u32(sm.v[st]), 8 * BN, kSwizzle128B);
#pragma unroll
                    for (int k = 0; k < BN / 32; ++k)   // UINT8 codes of keys 32k .. 32k + 31 at column 32k
                        mma_i8_ts(tO, tS + b * BN + 32 * k, vdesc + 2 * k, idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&sm.empty[st]);
                    mma_commit(&sm.pv_done[b]);
                    if (j == nb - 1) mma_commit(&sm.acc_full);
                }
                if (s + SB < T) ok = issue_qk(s + SB);
            }
            // Drain: every MMA issued has completed before TMEM is freed.
            mma_commit(&sm.mma_drain);
            drain_wait(&sm.mma_drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------ rows (warps 0-7) ---
        const int quad = warp & 3, half = warp >> 2;
        const int row = 32 * quad + lane;
        const int qi = q0 + row;
        const int lim = causal ? min(L, qi + 1) : L;
        const uint32_t lane_off = static_cast<uint32_t>(32 * quad) << 16;
        const int kofs = 32 * kChunks * half;   // this warp's keys in each block
        bool ok = true;
        uint32_t w[kChunks][32];
        // -- pass A: the integer row max over this half's visible keys (as a biased float)
        float mx[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int j = 0; j < nb; ++j) {
            const int s = j, b = s % SB;
            if (!warp_wait(&sm.s_full[b], (s / SB) & 1, abort_flag, 8)) { ok = false; break; }
            tc_fence_after();
            const uint32_t ts = tS + lane_off + b * BN + kofs;
#pragma unroll
            for (int ch = 0; ch < kChunks; ++ch) tmem_ld32(ts + 32 * ch, w[ch]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.s_read[b]);
            if ((causal && j == nb - 1) || ((j + 1) * BN > L)) {
#pragma unroll
                for (int ch = 0; ch < kChunks; ++ch) mask_zero(w[ch], j * BN + kofs + 32 * ch, lim);
            }
#pragma unroll
            for (int ch = 0; ch < kChunks; ++ch) max_chunk(w[ch], mx);
        }
        sm.half_max[half][row] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        row_barrier();
        float mbf = sm.half_max[0][row];
#pragma unroll
        for (int h = 1; h < kParts; ++h) mbf = fmaxf(mbf, sm.half_max[h][row]);
        // -- the head's clip threshold and index scale
        const long long cint = clip_threshold(c, D, __ldg(sQ + bh), __ldg(sK + bh));
        const bool fast = cint <= (1ll << (23 - bits));
        const float cf = cint < (1ll << 24) ? static_cast<float>(cint) : 16777216.0f;
        // q = (2^b - 1) / c_int rounded up: then floor(D' q) = floor(D' (2^b - 1) / c_int)
        // for every integer 0 <= D' <= c_int while c_int <= 2^(23 - b)
        const float q = __fdiv_ru(static_cast<float>(nm1), cf);
        // -- pass B: distances, table, P codes, integer row sum of this half
        uint32_t l = 0;
        for (int j = 0; ok && j < nb; ++j) {
            const int s = nb + j, b = s % SB;
            if (!warp_wait(&sm.s_full[b], (s / SB) & 1, abort_flag, 9)) { ok = false; break; }
            tc_fence_after();
            const uint32_t ts = tS + lane_off + b * BN + kofs;
#pragma unroll
            for (int ch = 0; ch < kChunks; ++ch) tmem_ld32(ts + 32 * ch, w[ch]);
            tmem_wait_ld();
            const bool need_mask = (causal && j == nb - 1) || ((j + 1) * BN > L);
            if (fast)
                lookup_block<true, kChunks>(w, mbf, cf, q, static_cast<unsigned long long>(cint), nm1, sm.lut,
                                      need_mask, j * BN + kofs, lim, l, ts);
            else
                lookup_block<false, kChunks>(w, mbf, cf, q, static_cast<unsigned long long>(cint), nm1, sm.lut,
                                       need_mask, j * BN + kofs, lim, l, ts);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_full[b]);
        }
        sm.half_sum[half][row] = l;
        row_barrier();
        uint32_t lrow = 0;
#pragma unroll
        for (int h = 0; h < kParts; ++h) lrow += sm.half_sum[h][row];
        // -- epilogue: O = s_V acc / l, each half writing D / 2 channels
        if (ok && warp_wait(&sm.acc_full, 0, abort_flag, 10)) {
            tc_fence_after();
            const float f = __ldg(sV + bh) / static_cast<float>(lrow);   // l >= 255 (the max key)
            const int64_t obase = (static_cast<int64_t>(bh) * L + qi) * D;
#pragma unroll
            for (int ch = half; ch < D / 32; ch += kParts) {
                uint32_t a[32];
                tmem_ld32(tO + lane_off + 32 * ch, a);
                tmem_wait_ld();
                if (qi < L) {
                    uint4 *dst = reinterpret_cast<uint4 *>(O + obase + 32 * ch);
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        uint4 wv;
                        __half2 *h = reinterpret_cast<__half2 *>(&wv);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            h[e] = __floats2half2_rn(__int2float_rn(static_cast<int32_t>(a[8 * c8 + 2 * e])) * f,
                                                     __int2float_rn(static_cast<int32_t>(a[8 * c8 + 2 * e + 1])) * f);
                        dst[c8] = wv;
                    }
                }
            }
            if (qi < L && half == 0) {
                const int64_t r = static_cast<int64_t>(bh) * L + qi;
                if (m_out) m_out[r] = __float2int_rn(mbf - kBias);
                if (l_out) l_out[r] = static_cast<int32_t>(lrow);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(sm.tmem_base, kTmemCols);
    }
}

// ----------------------------------------------------------- host side ---

template <int D>
int launch_index(const int8_t *Qq, const int8_t *Kq, const int8_t *Vt, const float *sQ, const float *sK,
                 const float *sV, int BH, int L, int causal, double c, int bits, void *O,
                 int32_t *m_out, int32_t *l_out, cudaStream_t stream) {
    const int64_t ld = intfa_vt_ld(L);
    const CUtensorMapSwizzle swz = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap mq, mk, mv;
    int rc = make_map(&mq, Qq, D, L, BH, D, static_cast<uint64_t>(L) * D, D, BM, swz);
    if (!rc) rc = make_map(&mk, Kq, D, L, BH, D, static_cast<uint64_t>(L) * D, D, BN, swz);
    if (!rc) rc = make_map(&mv, Vt, ld, D, BH, ld, static_cast<uint64_t>(ld) * D, BN, D,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    const size_t smem = idx_smem_bytes<D>();
    rc = cuda_status(cudaFuncSetAttribute(attn_index_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(smem)));
    if (rc) return rc;
    const dim3 grid(static_cast<unsigned>((L + BM - 1) / BM), static_cast<unsigned>(BH));
    attn_index_kernel<D><<<grid, kThreads, smem, stream>>>(mq, mk, mv, sQ, sK, sV, static_cast<__half *>(O), L,
                                                           causal, c, bits, m_out, l_out);
    return cuda_status(cudaGetLastError());
}

}  // namespace

int read_index_status(int clear, uint32_t *word) {
    uint32_t w = 0;
    int rc = cuda_status(cudaMemcpyFromSymbol(&w, g_status_index, sizeof(w)));
    if (rc) return rc;
    if (clear) {
        const uint32_t z = 0;
        rc = cuda_status(cudaMemcpyToSymbol(g_status_index, &z, sizeof(z)));
        if (rc) return rc;
    }
    *word = w;
    return INTFA_OK;
}

}  // namespace intfa

// ------------------------------------------------------------------ C ABI ---

extern "C" int intfa_index_attention_fwd(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                                         const float *s_Q, const float *s_K, const float *s_V, int B,
                                         int H, int L, int d, int causal, double c, int b, void *O_f16,
                                         int32_t *m_out, int32_t *l_out, void *stream) {
    using namespace intfa;
    if (B <= 0 || H <= 0 || L <= 0) return INTFA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    if (!(c > 0.0) || !(c < 1.0e30) || b < 1 || b > 8) return INTFA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return INTFA_ERR_UNSUPPORTED;
    if (L > 65536) return INTFA_ERR_UNSUPPORTED;   // int32 accumulation: 255 * 127 * L < 2^31
    const int64_t bh = static_cast<int64_t>(B) * H;
    if (bh > 65535) return INTFA_ERR_UNSUPPORTED;  // grid y
    if (!Q_q || !K_q || !Vt_q || !s_Q || !s_K || !s_V || !O_f16) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(Q_q) || !aligned16(K_q) || !aligned16(Vt_q) || !aligned16(O_f16) ||
        (reinterpret_cast<uintptr_t>(s_Q) & 3u) || (reinterpret_cast<uintptr_t>(s_K) & 3u) ||
        (reinterpret_cast<uintptr_t>(s_V) & 3u) || (reinterpret_cast<uintptr_t>(m_out) & 3u) ||
        (reinterpret_cast<uintptr_t>(l_out) & 3u))
        return INTFA_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d == 128)
        return launch_index<128>(Q_q, K_q, Vt_q, s_Q, s_K, s_V, static_cast<int>(bh), L, causal, c, b, O_f16,
                                 m_out, l_out, s);
    return launch_index<64>(Q_q, K_q, Vt_q, s_Q, s_K, s_V, static_cast<int>(bh), L, causal, c, b, O_f16, m_out,
                            l_out, s);
}
