// attention.cu -- fused INT8 attention forward pass for sm_100a.
//
// Method (INT-FlashAttention: Enabling Flash Attention for INT8 Quantization,
// abstract; IntAttention: A Fully Integer Attention Pipeline for Efficient
// Edge Inference, section 2.1 eqs. 4-5, section 2.2 eq. 6, section 3.2;
// FlashAttention-3, abstract, for the block-wise online softmax):
//   S_ij  = sum_k Q_hat[i,k] K_hat[j,k]                   INT8 x INT8 -> INT32
//   t_ij  = S_ij s_Q[i] s_K[j] / sqrt(d)                  (keys j > i masked if causal)
//   per key block of 128:  m_new = max(m, max_j t_ij), alpha = exp(m - m_new)
//                          p_ij = exp(t_ij - m_new),  P_hat = RNE(127 p_ij)
//                          acc  = alpha acc + P_hat V_hat   (INT8 x INT8 -> INT32)
//                          l    = alpha l + sum_j p_ij
//   O_i   = s_V acc_i / (127 l_i)                          -> fp16
// exp is evaluated as exp2 with log2(e) folded into the per-row constant.
//
// B200 design: a persistent kernel, one CTA per SM, each CTA walking a fixed
// list of 128-query tiles (tile c, c + G, c + 2G, ... of the head-major
// order).  Every role runs through the CTA's whole stream of (tile, key
// block) pairs with ring counters that do not restart at tile boundaries, so
// the loads and Q K^T of the next tile overlap the last blocks and the
// epilogue of the current one.  16 warps:
//   role 12     TMA producer: each tile's Q_hat (two Q buffers), K_hat tile,
//               V_hat tile and the block's s_K values into a 5-stage
//               shared-memory ring.  V_hat comes either as stored, [L][d]
//               (kVRow: the P V product reads the tile N-major), or
//               transposed, [d][Lv] (K-major).
//   role 13     tensor-core issuer (one lane): S = Q K^T with tcgen05.mma
//               kind::i8 into one of three TMEM S buffers, three key blocks
//               ahead of P V; P V with the P codes read straight from TMEM
//               (aliasing columns of the S buffer they came from) into the
//               TMEM int32 P V block; owns the TMEM allocation (S0..S2: 3 x
//               128 columns; P V block: 128 columns).  Before the INT8 MMAs
//               of a block, one fp16 MMA of constant operands sets the target
//               accumulator to a float bias (kBiasA), so that the readers
//               get exact fp32 values with one add instead of a conversion.
//   roles 0-7   softmax, two warpgroups taking alternate key blocks of the
//               stream (one thread per query row, all 128 keys of the
//               block): pass 1 v = S s_K (written back over S), causal /
//               ragged mask, row max; the running max m from the other
//               warpgroup's preceding block; alpha to the output side; pass 2
//               p = 2^(c v - c m), the row sum and the P codes, written back
//               to TMEM as the A operand of P V.  While one warpgroup is in
//               pass 2 (special-function bound) the other can run pass 1.
//   roles 8-11  output side (one thread per query row): folds each int32
//               P V block into the row's fp32 accumulator, held in registers
//               (o = alpha o + block), and writes the normalised fp16 row at
//               the end of each tile.
//   roles 14-15 the in-kernel Q quantiser (fp16 Q entry point), else idle.
// Roles 12-15 run on hardware warps 0-3, roles 0-11 on hardware warps 4-15;
// a role keeps its hardware warp's TMEM lane quadrant (role mod 4).
// Every wait is bounded (clock-based); a timeout records a status word,
// raises a CTA-wide abort flag, drains in-flight copies and MMAs, frees TMEM
// and returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include "internal.h"
#include "ptx.cuh"
#include "quant_math.cuh"
#include "tma_host.h"

namespace intfa {

__device__ uint32_t g_status;  // 0 = fine; else 0x100 | wait site of the first timeout

namespace {

constexpr int BM = 128;                       // query rows per CTA
constexpr int BN = 128;                       // keys per block
// K/V ring depth
template <bool kQ16>
constexpr int kv_stages() { return 5; }
constexpr int kQHalf = BM / 2;                // fp16 Q rows staged at a time (in-kernel quantiser)
constexpr int kThreads = 512;                 // 16 warps = 4 warpgroups
constexpr int SB = 3;                         // TMEM S buffers
constexpr int OB = 1;                         // TMEM P V blocks
constexpr int AB = 4;                         // alpha ring depth (softmax -> output side); even
// Register split (setmaxnreg): launched with kLaunchRegs per thread (checked
// on the host before every launch); the output warpgroup, which holds a
// d-column fp32 row, and the two softmax warpgroups take registers from the
// producer / MMA warpgroup.  The shares add up to at most the launch total.
constexpr int kLaunchRegs = 128;
template <int D, bool kQ16>
struct RegSplit {   // d = 128: the output row alone is 128 registers
    static constexpr uint32_t kSoft = 136;    // each of the two softmax warpgroups
    static constexpr uint32_t kOutput = 192;
    static constexpr uint32_t kOther = 48;    // also the in-kernel Q quantiser (roles 14, 15)
};
template <bool kQ16>
struct RegSplit<64, kQ16> {
    static constexpr uint32_t kSoft = 136;
    static constexpr uint32_t kOutput = 168;
    static constexpr uint32_t kOther = 72;
};
template <int D, bool kQ16>
constexpr bool split_fits() {
    using R = RegSplit<D, kQ16>;
    return 128 * (2 * R::kSoft + R::kOutput + R::kOther) <= kThreads * kLaunchRegs;
}
static_assert(split_fits<128, false>() && split_fits<64, false>() && split_fits<128, true>() &&
                  split_fits<64, true>(),
              "register split exceeds the launch allocation");
// Warp roles inside the fourth warpgroup (roles 12-15).
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kQuantWarp = 14;   // and 15
constexpr int kTmemCols = 512;

// Moves this warpgroup from kLaunchRegs to R registers per thread with the
// matching setmaxnreg direction (chosen at compile time).
template <uint32_t R>
__device__ __forceinline__ void regs_to() {
    static_assert(R % 8 == 0 && R >= 24 && R <= 256, "setmaxnreg range");
    if constexpr (R > static_cast<uint32_t>(kLaunchRegs)) regs_inc<R>();
    else if constexpr (R < static_cast<uint32_t>(kLaunchRegs)) regs_dec<R>();
}
constexpr long long kWaitCycles = 1ll << 32;  // ~2 s at B200 clocks (the release cap)
constexpr float kLog2e = 1.4426950408889634f;
// 1.5 * 2^23: for 0 <= y < 2^22, fl(y + 1.5 * 2^23) is 1.5 * 2^23 + RNE(y),
// so RNE(y) sits in the low mantissa bits of that float.
constexpr float kMagic = 12582912.0f;
// Accumulator bias.  Each S buffer and the P V block are first set to the
// fp32 value 1.5 * 2^23 (bit pattern 0x4B400000) by one fp16 MMA of constant
// operands (16 products 1024 * 768, all exact), and the INT8 MMAs then add
// their int32 results to that bit pattern.  For |x| < 2^22 the sum
// 0x4B400000 + x is the bit pattern of the float 1.5 * 2^23 + x, so an
// accumulator read as fp32 minus kMagic is exactly float(x): no int -> float
// conversion instruction is needed (|S| <= 127^2 d; |P V| per block <=
// 255 * 127 * 128 with UINT8 codes; both below 2^22).
constexpr uint16_t kBiasA = 0x6400;   // fp16 1024
constexpr uint16_t kBiasB = 0x6200;   // fp16 768
static_assert(255 * 127 * BN < (1 << 22) && 127 * 127 * 128 < (1 << 22), "biased accumulator range");

// (-kMagic, -kMagic) as an f32x2 operand, materialised where it is used (an
// opaque move, so that the compiler does not keep it in registers across
// the roles of the kernel).
__device__ __forceinline__ uint64_t neg_bias2() {
    uint64_t r;
    asm volatile("mov.b64 %0, 0xCB400000CB400000;" : "=l"(r));
    return r;
}

// -------------------------------------------------------- bounded waits ---

// A waiting thread sleeps inside try_wait (suspend-time hint) between probes.
constexpr uint32_t kSleepNs = 1000000;

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         uint32_t site, long long cap = kWaitCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity, kSleepNs)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > cap) {
            *abort_flag = 1;
            atomicCAS(&g_status, 0u, 0x100u | site);
            return false;
        }
    }
    return true;
}

// Warp-uniform bounded wait: every lane polls, the warp agrees on the result.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          uint32_t site, long long cap = kWaitCycles) {
    const bool ok = wait_bar(bar, parity, abort_flag, site, cap);
    return __all_sync(0xFFFFFFFFu, ok);
}

// Bounded wait that ignores the abort flag (used to drain in-flight work).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity, long long cap = kWaitCycles) {
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity, kSleepNs)) {
        if (clock64() - t0 > cap) {
            atomicCAS(&g_status, 0u, 0x1FFu);
            return;
        }
    }
}

// ------------------------------------------------------- shared memory ---

template <int D, bool kQ16>
struct alignas(1024) AttnSmem {
    static constexpr int NS = kv_stages<kQ16>();
    uint8_t q[2][BM * D];       // Q_hat tiles (two query tiles in flight), K-major, TMA-swizzled
    uint8_t qs[kQ16 ? kQHalf * D * 2 : 1024];   // half an fp16 Q tile for the in-kernel quantiser
    uint8_t k[NS][BN * D];      // K_hat tiles
    uint8_t v[NS][D * BN];      // V_hat tiles: 128 keys x D (kVRow) or D channels x 128 keys
    float sk[NS][BN];           // s_K of each key block
    float mrow[2][BM];          // softmax warpgroup w -> the other: running max after its latest block
    float alpha_o[AB][BM];      // softmax -> output: alpha of block g (slot g mod AB)
    float lsum[2][2][BM];       // softmax warpgroup w -> output: its share of the row sum (slot = tile mod 2)
    float cml[2][2][BM];        //   ... and c m at its last block of the tile (the share's reference)
    uint16_t bias_ab[2][192];   // fp16 operands of the bias MMA: 1024 (A), 768 (B)
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[NS], v_full[NS], kv_empty[NS];
    uint64_t s_full[SB], p_full[SB];
    uint64_t m_full[2][4];      // softmax warpgroup w, warp k: mrow[w] rows of quadrant k written
    uint64_t a_full[AB][4];     // softmax warp k -> output warp k
    uint64_t a_empty[AB][4];    // output warp k -> softmax warp k
    uint64_t o_full[OB], o_empty[OB];
    uint64_t l_full[2], l_empty[2];
    float sq[8][BM];            // in-kernel Q quantiser -> prep: s_Q of tile i (slot i mod 8)
    uint64_t sq_full[8];
    uint64_t qs_full, qs_empty; // fp16 Q staging: TMA -> quantiser warps -> next TMA
    uint64_t mma_drain;
    uint32_t tmem_base;
    int abort_flag;
};

template <int D, bool kQ16>
constexpr size_t attn_smem_bytes() {
    // 1024 for manual alignment; D = 64 is padded so that only one CTA (which
    // holds all 512 TMEM columns) is resident per SM.
    size_t s = sizeof(AttnSmem<D, kQ16>) + 1024;
    return s < 120 * 1024 ? 120 * 1024 : s;
}
static_assert(attn_smem_bytes<128, false>() <= 227 * 1024 && attn_smem_bytes<128, true>() <= 227 * 1024 &&
                  attn_smem_bytes<64, false>() <= 227 * 1024 && attn_smem_bytes<64, true>() <= 227 * 1024,
              "shared memory above the per-block limit");

// Dynamic shared memory rounded up to 1024 B by pointer arithmetic on the
// __shared__ array itself, so that the compiler keeps every access in the
// shared state space (an integer round trip would make them generic).
__device__ __forceinline__ uint8_t *smem_aligned_1024() {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t off = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    return smem_raw + off;
}

template <int D, bool kQ16>
__device__ __forceinline__ AttnSmem<D, kQ16> &get_smem() {
    return *reinterpret_cast<AttnSmem<D, kQ16> *>(smem_aligned_1024());
}

// ----------------------------------------------------------- tiles ---

// Query tiles in head-major order (a head's K_hat / V_hat then stay in L2
// while the CTAs working on it are resident), the heaviest causal tile of
// each head first.  CTA c processes tiles c, c + G, c + 2G, ... (G = grid).
struct Tile {
    int bh, q0, nb;   // head, first query row, key blocks
};

__device__ __forceinline__ Tile tile_at(int t, int ntiles, int L, int causal) {
    Tile r;
    r.bh = t / ntiles;
    const int tt = t - r.bh * ntiles;
    const int qt = causal ? (ntiles - 1 - tt) : tt;
    r.q0 = qt * BM;
    r.nb = causal ? (qt + 1) : (L + BN - 1) / BN;
    return r;
}

// Position in this CTA's stream of (tile, key block) pairs.
struct Cursor {
    int t, i, j;   // tile id (>= total when done), tile count so far, key block
    Tile T;
};

__device__ __forceinline__ Cursor cursor_begin(int ntiles, int total, int L, int causal) {
    Cursor c;
    c.t = blockIdx.x;
    c.i = 0;
    c.j = 0;
    c.T = c.t < total ? tile_at(c.t, ntiles, L, causal) : Tile{0, 0, 0};
    return c;
}

__device__ __forceinline__ void cursor_next(Cursor &c, int ntiles, int total, int L, int causal) {
    if (++c.j < c.T.nb) return;
    c.j = 0;
    ++c.i;
    c.t += gridDim.x;
    if (c.t < total) c.T = tile_at(c.t, ntiles, L, causal);
}

// Slot and phase parity of a ring of N mbarrier-guarded buffers, advanced one
// block at a time (block g: idx = g mod N, ph = (g / N) mod 2) without
// integer division.
template <int N>
struct Ring {
    int idx = 0;
    uint32_t ph = 0;
    __device__ __forceinline__ void next() {
        if (++idx == N) {
            idx = 0;
            ph ^= 1u;
        }
    }
    __device__ __forceinline__ Ring after() const {
        Ring r = *this;
        r.next();
        return r;
    }
};

// ------------------------------------------------------- prep pieces ---

// v = fl(S s_K) in place, from the biased accumulator (fl(x - kMagic) = S
// exactly).
__device__ __forceinline__ void scores_to_v(uint32_t (&w)[32], const float4 *sk4) {
    const uint64_t nb2 = neg_bias2();
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 k4 = sk4[q];
        const uint64_t a = fmul2(fadd2(f2_pack(__uint_as_float(w[4 * q]), __uint_as_float(w[4 * q + 1])), nb2),
                                 f2_pack(k4.x, k4.y));
        const uint64_t e = fmul2(fadd2(f2_pack(__uint_as_float(w[4 * q + 2]), __uint_as_float(w[4 * q + 3])), nb2),
                                 f2_pack(k4.z, k4.w));
        float v0, v1, v2, v3;
        f2_unpack(a, v0, v1);
        f2_unpack(e, v2, v3);
        w[4 * q] = __float_as_uint(v0);
        w[4 * q + 1] = __float_as_uint(v1);
        w[4 * q + 2] = __float_as_uint(v2);
        w[4 * q + 3] = __float_as_uint(v3);
    }
}

// Keys at or past lim get v = -inf.
__device__ __forceinline__ void mask_v(uint32_t (&w)[32], int key0, int lim) {
#pragma unroll
    for (int e = 0; e < 32; ++e)
        if (key0 + e >= lim) w[e] = __float_as_uint(-INFINITY);
}

__device__ __forceinline__ void max_v(const uint32_t (&w)[32], float (&mx)[4]) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        mx[q & 3] = fmax3(mx[q & 3], __uint_as_float(w[4 * q]), __uint_as_float(w[4 * q + 1]));
        mx[(q + 2) & 3] =
            fmax3(mx[(q + 2) & 3], __uint_as_float(w[4 * q + 2]), __uint_as_float(w[4 * q + 3]));
    }
}

// One 32-key chunk of v: p = 2^(c v - c m) (<= 1; 0 for masked keys), the
// running pair sums of p (or, kCodes, the integer sum of the P codes), and
// the 32 P codes RNE(127 p) packed four per word (the code is the low byte of
// fl(127 p + 1.5 * 2^23)).
template <bool kCodes>
__device__ __forceinline__ void exp_codes(const uint32_t (&w)[32], uint64_t c2, uint64_t ncm2, uint64_t k127,
                                          uint64_t magic, uint64_t &ps01, uint64_t &ps23, uint32_t (&pk)[8],
                                          uint32_t &csum) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float x0, x1, x2, x3;
        f2_unpack(ffma2(f2_pack(__uint_as_float(w[4 * q]), __uint_as_float(w[4 * q + 1])), c2, ncm2), x0, x1);
        f2_unpack(ffma2(f2_pack(__uint_as_float(w[4 * q + 2]), __uint_as_float(w[4 * q + 3])), c2, ncm2), x2, x3);
        const uint64_t p01 = f2_pack(ex2(x0), ex2(x1));
        const uint64_t p23 = f2_pack(ex2(x2), ex2(x3));
        if constexpr (!kCodes) {
            ps01 = fadd2(ps01, p01);
            ps23 = fadd2(ps23, p23);
        }
        float t0, t1, t2, t3;
        f2_unpack(ffma2(p01, k127, magic), t0, t1);
        f2_unpack(ffma2(p23, k127, magic), t2, t3);
        pk[q] = prmt(prmt(__float_as_uint(t0), __float_as_uint(t1), 0x0040u),
                     prmt(__float_as_uint(t2), __float_as_uint(t3), 0x0040u), 0x5410u);
        if constexpr (kCodes) csum = __dp4a(pk[q], 0x01010101u, csum);
    }
}

// ---------------------------------------------------------------- kernel ---

// kQ16: Q arrives as fp16 (Qh) and is quantised per token inside the kernel
// by roles 14-15 (bit-identical to quant_per_token_kernel); its scales go to
// the softmax warps through shared memory and, if sQ_out is set, to global.
// Otherwise Q_hat arrives through tmQ and s_Q through sQ.
// kLCodes: the row sum from the P codes, l = alpha l + sum_j P_hat_ij / 127,
// instead of the unquantised p (the other reading of the pages).
// kU8P: P codes RNE(255 p) stored as UINT8 and multiplied as unsigned A
// operands (IntAttention Table 5's unsigned scheme; |P V| per block <=
// 255 * 127 * 128 < 2^22 keeps the biased accumulator exact); 127 becomes 255
// in the code rounding, the code sum and the epilogue.
// kDbg (test forms): 0 release; 1 also writes the recovered S of every block
// (exact int32, from the biased accumulator) to dbg[bh][query][key]; 2 issues
// no load and no MMA, so that every wait runs out after `cap` clock cycles
// (the timeout path).  `cap` bounds every wait of the kernel's roles.
template <int D, bool kQ16, bool kLCodes = false, bool kU8P = false, int kDbg = 0, bool kVRow = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const float *__restrict__ sQ,
                    const float *__restrict__ sK, const float *__restrict__ sV,
                    __half *__restrict__ O, int BH, int L, int causal,
                    const uint4 *__restrict__ Qh, float *__restrict__ sQ_out, int sshift, long long cap,
                    int32_t *__restrict__ dbg) {
    AttnSmem<D, kQ16> &sm = get_smem<D, kQ16>();
    constexpr int NS = AttnSmem<D, kQ16>::NS;
    // every wait's cap: the release constant, or the test form's argument
    const long long wcap = kDbg == 2 ? cap : kWaitCycles;
    constexpr float kLevels = kU8P ? 255.0f : 127.0f;   // largest P code
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    // Role numbering: the producer / MMA warpgroup (roles 12-15) runs on the
    // lowest hardware warps 0-3, which the warp schedulers favour, so that the
    // issue of tensor-core work is not queued behind the compute warps.  A
    // role keeps its hardware warp's TMEM lane quadrant (role mod 4).
    const int hw_warp = tid >> 5;
    const int warp = hw_warp < 4 ? hw_warp + 12 : hw_warp - 4;
    const int rtid = 32 * warp + lane;

    const int ntiles = (L + BM - 1) / BM;
    const int total = BH * ntiles;
    volatile int *abort_flag = &sm.abort_flag;

    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.q_full[b], kQ16 ? 64 : 1);
            mbar_init(&sm.q_empty[b], 1);
            mbar_init(&sm.l_full[b], 2 * BM);
            mbar_init(&sm.l_empty[b], BM);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.k_full[s], 32);
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.kv_empty[s], 1 + BM);
        }
        for (int b = 0; b < SB; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.p_full[b], BM);
        }
        for (int w = 0; w < 2; ++w)
            for (int k = 0; k < 4; ++k) mbar_init(&sm.m_full[w][k], 32);
        for (int b = 0; b < AB; ++b)
            for (int k = 0; k < 4; ++k) {
                mbar_init(&sm.a_full[b][k], 32);
                mbar_init(&sm.a_empty[b][k], 32);
            }
        for (int b = 0; b < OB; ++b) {
            mbar_init(&sm.o_full[b], 1);
            mbar_init(&sm.o_empty[b], BM);
        }
        for (int b = 0; b < 8; ++b) mbar_init(&sm.sq_full[b], 64);
        mbar_init(&sm.qs_full, 1);
        mbar_init(&sm.qs_empty, 64);
        mbar_init(&sm.mma_drain, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (tid < 2 * 192) {
        sm.bias_ab[tid / 192][tid % 192] = tid < 192 ? kBiasA : kBiasB;
        fence_proxy_async_smem();   // read by the tensor core
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;
    const uint32_t tS = tbase;              // S buffer s at column 128 s
    const uint32_t tO = tbase + 128 * SB;   // int32 P V block o at column tO + 128 o

    if (warp >= 12) {
      regs_to<RegSplit<D, kQ16>::kOther>();
      if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer ---
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
        }
        // s_K of a key block as four floats per lane (zero past the end);
        // the loads for the next block are issued one block ahead so that
        // their latency overlaps the wait for a free stage.
        // With scale blocks of 2^sshift tokens (sshift = 0: one scale per
        // token) the scale of key j is s_K[j >> sshift].
        const int64_t nsc = (static_cast<int64_t>(L) + (1 << sshift) - 1) >> sshift;
        auto load_sk = [&](const Cursor &c) {
            const float *src = sK + static_cast<int64_t>(c.T.bh) * nsc;
            const int key = c.j * BN + 4 * lane;
            float4 v4;
            v4.x = key + 0 < L ? __ldg(src + ((key + 0) >> sshift)) : 0.0f;
            v4.y = key + 1 < L ? __ldg(src + ((key + 1) >> sshift)) : 0.0f;
            v4.z = key + 2 < L ? __ldg(src + ((key + 2) >> sshift)) : 0.0f;
            v4.w = key + 3 < L ? __ldg(src + ((key + 3) >> sshift)) : 0.0f;
            return v4;
        };
        Cursor c = cursor_begin(ntiles, total, L, causal);
        float4 sk_next = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (c.t < total) sk_next = load_sk(c);
        int g = 0, q_issued = 0;
        Ring<NS> kv;
        while (kDbg != 2 && c.t < total) {
            if (!kQ16 && c.j == 0) {   // a new tile: its Q_hat into buffer i mod 2
                const int qb = c.i & 1;
                if (c.i >= 2 && !warp_wait(&sm.q_empty[qb], ((c.i >> 1) - 1) & 1, abort_flag, 8, wcap)) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sm.q_full[qb], BM * D);
                    tma_load_3d(&tmQ, &sm.q_full[qb], sm.q[qb], 0, c.T.q0, c.T.bh);
                }
                q_issued = c.i + 1;
            }
            const int st = kv.idx;
            if (g >= NS && !warp_wait(&sm.kv_empty[st], kv.ph ^ 1u, abort_flag, 1, wcap)) break;
            if (lane == 0) {
                mbar_expect_tx(&sm.k_full[st], BN * D);
                tma_load_3d(&tmK, &sm.k_full[st], sm.k[st], 0, c.j * BN, c.T.bh);
                mbar_arrive_expect_tx(&sm.v_full[st], D * BN);
                if constexpr (kVRow)   // BN rows of V_hat, D bytes each
                    tma_load_3d(&tmV, &sm.v_full[st], sm.v[st], 0, c.j * BN, c.T.bh);
                else                   // D rows of V_hat^T, BN bytes each
                    tma_load_3d(&tmV, &sm.v_full[st], sm.v[st], c.j * BN, 0, c.T.bh);
            }
            *reinterpret_cast<float4 *>(&sm.sk[st][4 * lane]) = sk_next;
            mbar_arrive(&sm.k_full[st]);   // 32 arrivals + the K tile's bytes
            cursor_next(c, ntiles, total, L, causal);
            if (c.t < total) sk_next = load_sk(c);
            __syncwarp();
            ++g;
            kv.next();
        }
        // Drain: the last load issued into each stage and Q buffer has landed.
        for (int b = 0; !kQ16 && b < 2 && b < q_issued; ++b) {
            const int last = b + ((q_issued - 1 - b) / 2) * 2;
            drain_wait(&sm.q_full[b], (last >> 1) & 1, wcap);
        }
        for (int s = 0; s < NS && s < g; ++s) {
            const int last = s + ((g - 1 - s) / NS) * NS;   // last block using stage s
            drain_wait(&sm.k_full[s], (last / NS) & 1, wcap);
            drain_wait(&sm.v_full[s], (last / NS) & 1, wcap);
        }
        __syncwarp();
      } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer ---
        constexpr uint32_t kSwQK = (D == 128) ? kSwizzle128B : kSwizzle64B;
        constexpr uint32_t kSboQK = 8 * D;      // 8 rows of D bytes
        const uint32_t idesc_qk = make_idesc_i8(BM, BN);
        // kVRow: B = the V_hat tile as stored, [BN keys][D], read N-major
        // (bit 16 of the instruction descriptor: B is MN-major)
        const uint32_t idesc_pv = (kU8P ? make_idesc_u8s8(BM, D) : make_idesc_i8(BM, D)) | (kVRow ? (1u << 16) : 0u);
        // bias MMA operands: every element of A and B is the same constant, so
        // the descriptors may let core matrices overlap (16-byte strides keep
        // all reads inside the 384-byte arrays)
        const uint32_t idesc_bias_s = make_idesc_f16(BM, BN);
        const uint32_t idesc_bias_o = make_idesc_f16(BM, D);
        const uint64_t bias_a = make_sdesc_noswz(smem_u32(sm.bias_ab[0]), 16, 16);
        const uint64_t bias_b = make_sdesc_noswz(smem_u32(sm.bias_ab[1]), 16, 16);
        bool ok = true, issued = false;
        // qc walks the blocks whose Q K^T is issued, SB blocks ahead of pc,
        // which walks the blocks whose P V is issued.
        Cursor qc = cursor_begin(ntiles, total, L, causal);
        Cursor pc = qc;
        int gq = 0;
        Ring<NS> q_st, p_st;   // K/V stage of the Q K^T / P V block
        Ring<SB> q_sb, p_sb;   // S buffer of the Q K^T / P V block
        uint32_t p_oph = 0;    // o_full / o_empty parity of the P V block (one P V block)
        auto issue_qk = [&]() -> bool {   // Q K^T of block gq (cursor qc) into S buffer gq mod SB
            const int qb = qc.i & 1, st = q_st.idx, sb = q_sb.idx;
            if (qc.j == 0 && !warp_wait(&sm.q_full[qb], (qc.i >> 1) & 1, abort_flag, 2, wcap)) return false;
            if (!warp_wait(&sm.k_full[st], q_st.ph, abort_flag, 6, wcap)) return false;
            tc_fence_after();
            if constexpr (kDbg == 2) issued = true;
            if (lane == 0) {
                const uint64_t qdesc = make_sdesc(smem_u32(sm.q[qb]), kSboQK, kSwQK);
                const uint64_t kdesc = make_sdesc(smem_u32(sm.k[st]), kSboQK, kSwQK);
                mma_f16_ss(tS + sb * BN, bias_a, bias_b, idesc_bias_s, 0);
#pragma unroll
                for (int k = 0; k < D / 32; ++k)
                    mma_i8_ss(tS + sb * BN, qdesc + 2 * k, kdesc + 2 * k, idesc_qk, 1);
                mma_commit(&sm.s_full[sb]);
                if (qc.j == qc.T.nb - 1) mma_commit(&sm.q_empty[qb]);   // last use of this Q tile
            }
            __syncwarp();
            cursor_next(qc, ntiles, total, L, causal);
            ++gq;
            q_st.next();
            q_sb.next();
            return true;
        };
        // Q K^T runs SB blocks ahead of P V: Q K^T of block g + SB reuses the
        // S buffer of block g and is issued right after P V of block g, which
        // the tensor pipe executes first.  Across a tile boundary this issues
        // the next tile's first Q K^T while the current tile finishes.
        while (ok && qc.t < total && gq < SB) ok = issue_qk();
        static_assert(OB == 1, "one P V block");
        bool first_pv = true;
        while (ok && pc.t < total) {
            const int st = p_st.idx, sb = p_sb.idx;
            if (!warp_wait(&sm.v_full[st], p_st.ph, abort_flag, 4, wcap)) break;
            // the P V block held the previous block: its output fold has read it
            if (!first_pv && !warp_wait(&sm.o_empty[0], p_oph ^ 1u, abort_flag, 5, wcap)) break;
            if (!warp_wait(&sm.p_full[sb], p_sb.ph, abort_flag, 3, wcap)) break;
            tc_fence_after();
            if (lane == 0) {
                // K-major V_hat^T: 8-row groups of BN bytes, keys 32k.. at byte 32k
                // of each row.  N-major V_hat: the swizzle atom is 8 keys x D
                // bytes (one atom spans N = D), atoms 8 D bytes apart along K,
                // keys 32k.. start 32 k D bytes into the tile.
                const uint64_t vdesc = kVRow ? make_sdesc(smem_u32(sm.v[st]), kSboQK, kSwQK)
                                             : make_sdesc(smem_u32(sm.v[st]), 8 * BN, kSwizzle128B);
                constexpr uint64_t kVStep = kVRow ? (32 * D) >> 4 : 32 >> 4;   // 16-byte units
                mma_f16_ss(tO, bias_a, bias_b, idesc_bias_o, 0);
#pragma unroll
                for (int k = 0; k < BN / 32; ++k)   // codes of keys 32k .. 32k + 31 at column 32k
                    mma_i8_ts(tO, tS + sb * BN + 32 * k, vdesc + kVStep * k, idesc_pv, 1);
                mma_commit(&sm.o_full[0]);
                mma_commit(&sm.kv_empty[st]);
            }
            __syncwarp();
            cursor_next(pc, ntiles, total, L, causal);
            first_pv = false;
            p_st.next();
            p_sb.next();
            p_oph ^= 1u;
            if (qc.t < total) ok = issue_qk();
        }
        // Drain: every MMA this warp issued has completed before TMEM is freed
        // (nothing to wait for if it never issued one).
        if (kDbg != 2 || issued) {
            if (lane == 0) mma_commit(&sm.mma_drain);
            __syncwarp();
            drain_wait(&sm.mma_drain, 0, wcap);
        }
        __syncwarp();
      }
      else if (kQ16) {
        // ------------------------------------------ Q quantiser (14, 15) ---
        // G lanes per row of D fp16 (8 per lane); the two warps take row
        // slices alternately.  Codes go straight into the swizzled K-major
        // layout the TMA would have produced (128-byte swizzle for D = 128:
        // 16-byte chunk k of row r at k ^ (r mod 8); 64-byte for D = 64:
        // chunk k at k ^ ((r / 2) mod 4)).
        constexpr int G = D / 8;
        constexpr int kRowsPerWarp = 32 / G;
        const int wq = warp - kQuantWarp, sub = lane % G;
        bool ok = true;
        for (int i = 0, t = blockIdx.x; ok && t < total; ++i, t += gridDim.x) {
            const Tile T = tile_at(t, ntiles, L, causal);
            const int qb = i & 1, ss = i & 7;
            // buffer qb held tile i - 2: its last Q K^T has been issued and run
            if (i >= 2 && !warp_wait(&sm.q_empty[qb], ((i >> 1) - 1) & 1, abort_flag, 18)) break;
            const uint32_t qbase = smem_u32(sm.q[qb]);
            const uint4 *stage = reinterpret_cast<const uint4 *>(sm.qs);
            // the tile's fp16 rows in two halves of kQHalf rows through the
            // staging buffer: warp 14 issues the TMA once both warps have
            // read the previous half
            for (int h = 0; ok && h < 2; ++h) {
                const int n = 2 * i + h;
                if (wq == 0) {
                    if (n >= 1 && !warp_wait(&sm.qs_empty, (n - 1) & 1, abort_flag, 21)) { ok = false; break; }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&sm.qs_full, kQHalf * D * 2);
                        tma_load_3d(&tmQ, &sm.qs_full, sm.qs, 0, T.q0 + kQHalf * h, T.bh);
                    }
                    __syncwarp();
                }
                if (!warp_wait(&sm.qs_full, n & 1, abort_flag, 20)) { ok = false; break; }
                for (int rr = wq * kRowsPerWarp; rr < kQHalf; rr += 2 * kRowsPerWarp) {
                    const int rs = rr + lane / G;   // row in the staging half
                    const int r = kQHalf * h + rs;  // row in the tile
                    const int qi = T.q0 + r;
                    float f[8];
                    qmath::unpack8(stage[rs * G + sub], f);   // rows past L were zero-filled by TMA
                    float amax = qmath::absmax8(f);
#pragma unroll
                    for (int o = G / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
                    const float s = qmath::div127(amax);
                    const uint2 w = qmath::codes8(f, s, qmath::rcp_or_zero(s));
                    const int ch = sub >> 1;   // 16-byte chunk of bytes 8 sub .. 8 sub + 7
                    const uint32_t sw = D == 128 ? static_cast<uint32_t>(r & 7) : static_cast<uint32_t>((r >> 1) & 3);
                    const uint32_t addr = qbase + static_cast<uint32_t>(r * D) +
                                          ((static_cast<uint32_t>(ch) ^ sw) << 4) + 8u * static_cast<uint32_t>(sub & 1);
                    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(w.x), "r"(w.y) : "memory");
                    if (sub == 0) {
                        sm.sq[ss][r] = s;
                        if (sQ_out != nullptr && qi < L) sQ_out[static_cast<int64_t>(T.bh) * L + qi] = s;
                    }
                }
                mbar_arrive(&sm.qs_empty);   // this half has been read
            }
            if (!ok) break;
            fence_proxy_async_smem();   // codes visible to the tensor core
            mbar_arrive(&sm.q_full[qb]);
            mbar_arrive(&sm.sq_full[ss]);
        }
      }
      // otherwise the other two warps of this warpgroup have no role
    } else if (warp < 8) {
        regs_to<RegSplit<D, kQ16>::kSoft>();
        // --------------------------------------------------- softmax ---
        // Warpgroup ws takes the blocks g = ws, ws + 2, ... of this CTA's
        // stream of (tile, key block) pairs; its warp quad holds TMEM lane
        // quadrant quad (query rows 32 quad .. 32 quad + 31).
        const int ws = warp >> 2, quad = warp & 3;
        const int row = 32 * quad + lane;
        const uint32_t lane_off = static_cast<uint32_t>(32 * quad) << 16;
        const uint64_t k127 = f2_pack(kLevels, kLevels), magic = f2_pack(kMagic, kMagic);
        bool ok = true;
        int g = 0;
        Ring<SB> sb;
        Ring<NS> ks;
        Ring<AB> as;
        for (int i = 0, t = blockIdx.x; ok && t < total; ++i, t += gridDim.x) {
            const Tile T = tile_at(t, ntiles, L, causal);
            const int qi = T.q0 + row;
            float s_q;
            if constexpr (kQ16) {
                // slot i mod 8 cannot be rewritten before this read: the
                // quantiser runs at most two tiles ahead of Q K^T, which runs
                // at most SB = 3 blocks ahead of this warp
                if (!warp_wait(&sm.sq_full[i & 7], (i >> 3) & 1, abort_flag, 19)) break;
                s_q = sm.sq[i & 7][row];
            } else {
                const int64_t nsc = (static_cast<int64_t>(L) + (1 << sshift) - 1) >> sshift;
                s_q = qi < L ? __ldg(sQ + static_cast<int64_t>(T.bh) * nsc + (qi >> sshift)) : 0.0f;
            }
            // c = s_Q[i] log2(e) / sqrt(d), so that t_ij log2(e) = c (S_ij s_K[j]).
            // Clamped to a tiny positive value: a zero Q row then still maps masked
            // keys (v = -inf) to p = 0 and visible keys to p = 1.
            const float c = fmaxf(s_q * (kLog2e / sqrtf(static_cast<float>(D))), 1e-30f);
            const uint64_t c2 = f2_pack(c, c);
            const int lim = causal ? min(L, qi + 1) : L;
            float l = 0.0f;              // this warpgroup's share of the row sum, relative to m_own
            float m_own = -INFINITY;     // running max after this warpgroup's latest block of the tile
            for (int j = 0; j < T.nb; ++j, ++g, sb.next(), ks.next(), as.next()) {
                if ((g & 1) != ws) continue;
                const int b = sb.idx, st = ks.idx, ab = as.idx;
                if (!warp_wait(&sm.s_full[b], sb.ph, abort_flag, 12, wcap)) { ok = false; break; }
                // s_K of this block: published by the producer's release-arrive
                if (!warp_wait(&sm.k_full[st], ks.ph, abort_flag, 13, wcap)) { ok = false; break; }
                tc_fence_after();
                const uint32_t ts = tS + lane_off + b * BN;
                const float4 *sk4 = reinterpret_cast<const float4 *>(sm.sk[st]);
                const bool need_mask = (causal && j == T.nb - 1) || ((j + 1) * BN > L);
                // -- pass 1: v = fl(S s_K) (written back over S), mask, row max;
                // two 32-column chunks in flight per load
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    uint32_t w0[32], w1[32];
                    tmem_ld32(ts + 64 * h, w0);
                    tmem_ld32(ts + 64 * h + 32, w1);
                    tmem_wait_ld();
                    if constexpr (kDbg == 1) {   // S as recovered from the biased accumulator
                        if (qi < L) {
                            int32_t *dst = dbg + (static_cast<int64_t>(T.bh) * L + qi) * L + j * BN + 64 * h;
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                if (j * BN + 64 * h + e < L)
                                    dst[e] = static_cast<int32_t>(__uint_as_float(w0[e]) - kMagic);
                                if (j * BN + 64 * h + 32 + e < L)
                                    dst[32 + e] = static_cast<int32_t>(__uint_as_float(w1[e]) - kMagic);
                            }
                        }
                    }
                    scores_to_v(w0, sk4 + 16 * h);
                    scores_to_v(w1, sk4 + 16 * h + 8);
                    // keys past the end of the sequence, or after the query
                    // (causal), get v = -inf (p = 0)
                    if (need_mask) {
                        mask_v(w0, j * BN + 64 * h, lim);
                        mask_v(w1, j * BN + 64 * h + 32, lim);
                    }
                    max_v(w0, mx);
                    max_v(w1, mx);
                    tmem_st32(ts + 64 * h, w0);
                    tmem_st32(ts + 64 * h + 32, w1);
                }
                mbar_arrive(&sm.kv_empty[st]);   // done with this block's s_K
                // running max through block g - 1 (the other warpgroup's); the
                // wait also orders this warpgroup's mrow write after the other's
                // read of the previous value
                float m_prev = -INFINITY;
                if (g > 0) {
                    if (!warp_wait(&sm.m_full[ws ^ 1][quad], ((g - 1) >> 1) & 1, abort_flag, 15, wcap)) {
                        ok = false;
                        break;
                    }
                    if (j > 0) m_prev = sm.mrow[ws ^ 1][row];
                }
                const float m_new = fmaxf(m_prev, fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])));
                sm.mrow[ws][row] = m_new;
                mbar_arrive(&sm.m_full[ws][quad]);
                const float alpha = ex2(c * (m_prev - m_new));    // 0 for the tile's first block
                const float lscale = ex2(c * (m_own - m_new));    // 0 for this warpgroup's first
                m_own = m_new;
                // alpha of block g -> the output warp of this quadrant (slot
                // g mod AB was last used by block g - AB, also this warpgroup's)
                if (g >= AB && !warp_wait(&sm.a_empty[ab][quad], as.ph ^ 1u, abort_flag, 14, wcap)) {
                    ok = false;
                    break;
                }
                sm.alpha_o[ab][row] = alpha;
                mbar_arrive(&sm.a_full[ab][quad]);
                tmem_wait_st();   // v is in TMEM before pass 2 reads it back
                // -- pass 2: p = 2^(c v - c m), row sum, P codes; the codes of
                // keys 32 k .. 32 k + 31 go to columns 32 k .. 32 k + 7 (already
                // read), the A operand of the k-th P V step
                const float cm = c * m_new;
                const uint64_t ncm2 = f2_pack(-cm, -cm);
                uint64_t ps01 = 0ull, ps23 = 0ull;
                uint32_t csum = 0;
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    uint32_t w0[32], w1[32];
                    tmem_ld32(ts + 64 * h, w0);
                    tmem_ld32(ts + 64 * h + 32, w1);
                    tmem_wait_ld();
                    uint32_t pk0[8], pk1[8];
                    exp_codes<kLCodes>(w0, c2, ncm2, k127, magic, ps01, ps23, pk0, csum);
                    exp_codes<kLCodes>(w1, c2, ncm2, k127, magic, ps01, ps23, pk1, csum);
                    tmem_st8(ts + 64 * h, pk0);
                    tmem_st8(ts + 64 * h + 32, pk1);
                }
                float bsum;
                if constexpr (kLCodes) {
                    bsum = static_cast<float>(csum) * (1.0f / kLevels);
                } else {
                    float ps0, ps1, ps2, ps3;
                    f2_unpack(ps01, ps0, ps1);
                    f2_unpack(ps23, ps2, ps3);
                    bsum = (ps0 + ps1) + (ps2 + ps3);
                }
                l = l * lscale + bsum;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&sm.p_full[b]);
            }
            if (!ok) break;
            // this tile's share of the row sum -> the output side (slot = tile
            // mod 2); c m_own is -inf if this warpgroup had no block of the tile
            const int ls = i & 1;
            if (i >= 2 && !warp_wait(&sm.l_empty[ls], ((i >> 1) - 1) & 1, abort_flag, 17, wcap)) break;
            sm.lsum[ls][ws][row] = l;
            sm.cml[ls][ws][row] = c * m_own;
            mbar_arrive(&sm.l_full[ls]);
        }
    } else {
        regs_to<RegSplit<D, kQ16>::kOutput>();
        // ------------------------------------------------ output side ---
        const int row = rtid - 256;
        const int quad = warp - 8;
        const uint32_t lane_off = static_cast<uint32_t>(32 * quad) << 16;
        bool ok = true;
        Ring<AB> as;
        uint32_t oph = 0;   // o_full parity (one P V block)
        for (int i = 0, t = blockIdx.x; ok && t < total; ++i, t += gridDim.x) {
            const Tile T = tile_at(t, ntiles, L, causal);
            const int qi = T.q0 + row;
            const float s_v = __ldg(sV + T.bh);   // needed at the tile's end; loaded early
            uint64_t o2[D / 2];   // the output row as fp32 pairs
#pragma unroll
            for (int e = 0; e < D / 2; ++e) o2[e] = 0ull;
            for (int j = 0; j < T.nb; ++j, as.next(), oph ^= 1u) {
                const int ab = as.idx;
                // o = alpha o + (P V block), the biased block turned into fp32
                // exactly (fl(x - kMagic), |P V| <= 127^2 128 < 2^22)
                const uint32_t to = tO;
                if (!warp_wait(&sm.o_full[0], oph, abort_flag, 9, wcap)) { ok = false; break; }
                if (!warp_wait(&sm.a_full[ab][quad], as.ph, abort_flag, 10, wcap)) { ok = false; break; }
                tc_fence_after();
                const float alpha = sm.alpha_o[ab][row];
                mbar_arrive(&sm.a_empty[ab][quad]);
                const uint64_t a2 = f2_pack(alpha, alpha);
                // x - kMagic as fma(x, 1, -kMagic) (exact; compiles to fewer
                // registers than the add form here)
                const uint64_t nb2 = neg_bias2();
                const uint64_t one2 = f2_pack(1.0f, 1.0f);
                // the block in pairs of 32-column chunks; once the last pair is
                // in registers the P V block is released for the next block
#pragma unroll
                for (int pr = 0; pr < D / 64; ++pr) {
                    uint32_t w0[32], w1[32];
                    tmem_ld32(to + lane_off + 64 * pr, w0);
                    tmem_ld32(to + lane_off + 64 * pr + 32, w1);
                    tmem_wait_ld();
                    if (pr == D / 64 - 1) {
                        tc_fence_before();
                        mbar_arrive(&sm.o_empty[0]);
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const uint64_t x = ffma2(f2_pack(__uint_as_float(w0[2 * e]), __uint_as_float(w0[2 * e + 1])), one2, nb2);
                        o2[32 * pr + e] = ffma2(o2[32 * pr + e], a2, x);
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const uint64_t x = ffma2(f2_pack(__uint_as_float(w1[2 * e]), __uint_as_float(w1[2 * e + 1])), one2, nb2);
                        o2[32 * pr + 16 + e] = ffma2(o2[32 * pr + 16 + e], a2, x);
                    }
                }
            }
            if (!ok) break;
            // the tile's row sum from the two softmax warpgroups' shares, each
            // rescaled from its own reference c m_w to the final one (the
            // larger: the running max only grows) -> normalised fp16 row
            const int ls = i & 1;
            if (!warp_wait(&sm.l_full[ls], (i >> 1) & 1, abort_flag, 11, wcap)) break;
            const float cm0 = sm.cml[ls][0][row], cm1 = sm.cml[ls][1][row];
            const float cmf = fmaxf(cm0, cm1);
            const float l = sm.lsum[ls][0][row] * ex2(cm0 - cmf) + sm.lsum[ls][1][row] * ex2(cm1 - cmf);
            mbar_arrive(&sm.l_empty[ls]);
            if (qi < L) {
                const float f = s_v / (kLevels * l);
                uint4 *dst = reinterpret_cast<uint4 *>(O + (static_cast<int64_t>(T.bh) * L + qi) * D);
#pragma unroll
                for (int c8 = 0; c8 < D / 8; ++c8) {
                    uint4 wv;
                    __half2 *h = reinterpret_cast<__half2 *>(&wv);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float lo, hi;
                        f2_unpack(o2[4 * c8 + e], lo, hi);
                        h[e] = __floats2half2_rn(lo * f, hi * f);
                    }
                    dst[c8] = wv;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// ------------------------------------------------------- debug Q K^T ---

template <int D>
struct alignas(1024) QKSmem {
    uint8_t q[BM * D];
    uint8_t k[BN * D];
    uint64_t full, done;
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(128, 1)
    debug_qk_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    int L, int32_t *__restrict__ S) {
    QKSmem<D> &sm = *reinterpret_cast<QKSmem<D> *>(smem_aligned_1024());
    const int tid = threadIdx.x, warp = tid >> 5;
    const int q0 = blockIdx.x * BM, k0 = blockIdx.y * BN, bh = blockIdx.z;
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) {
        mbar_init(&sm.full, 1);
        mbar_init(&sm.done, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;
    if (tid == 0) {
        mbar_arrive_expect_tx(&sm.full, BM * D + BN * D);
        tma_load_3d(&tmQ, &sm.full, sm.q, 0, q0, bh);
        tma_load_3d(&tmK, &sm.full, sm.k, 0, k0, bh);
    }
    bool ok = warp_wait(&sm.full, 0, abort_flag, 20);
    tc_fence_after();
    if (tid == 0 && ok) {
        constexpr uint32_t kSw = (D == 128) ? kSwizzle128B : kSwizzle64B;
        const uint64_t qd = make_sdesc(smem_u32(sm.q), 8 * D, kSw);
        const uint64_t kd = make_sdesc(smem_u32(sm.k), 8 * D, kSw);
#pragma unroll
        for (int k = 0; k < D / 32; ++k) mma_i8_ss(tbase, qd + 2 * k, kd + 2 * k, make_idesc_i8(BM, BN), k > 0);
        mma_commit(&sm.done);
    }
    if (!ok) {
        drain_wait(&sm.full, 0);
    } else if (warp_wait(&sm.done, 0, abort_flag, 21)) {
        tc_fence_after();
        const int qi = q0 + tid;
        const uint32_t lane_off = static_cast<uint32_t>(32 * warp) << 16;
#pragma unroll
        for (int ch = 0; ch < BN / 32; ++ch) {
            uint32_t r[32];
            tmem_ld32(tbase + lane_off + 32 * ch, r);
            tmem_wait_ld();
            if (qi < L) {
                int32_t *dst = S + (static_cast<int64_t>(bh) * L + qi) * L + k0 + 32 * ch;
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    if (k0 + 32 * ch + c < L) dst[c] = static_cast<int32_t>(r[c]);
            }
        }
    } else if (tid == 0) {
        // the MMA may still be in flight: wait for it before freeing TMEM
        drain_wait(&sm.done, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 128);
    }
}

// ----------------------------------------------------------- host side ---

// Grid of the persistent attention kernel: one CTA per SM.  CTA c takes tiles
// c, c + G, ...; with causal masking the per-tile work cycles with period
// ntiles inside each head, so G is chosen coprime to ntiles, which makes every
// CTA's tiles cover the heavy and light positions alike (one SM may idle).
unsigned persistent_grid(int64_t total, int ntiles, int causal, int nsm) {
    if (nsm < 1) nsm = 1;
    if (total <= nsm) return static_cast<unsigned>(total);
    int g = nsm;
    if (causal) {
        for (int cand = nsm; cand > nsm / 2; --cand) {
            int a = cand, b = ntiles;
            while (b) { const int r = a % b; a = b; b = r; }
            if (a == 1) { g = cand; break; }
        }
    }
    return static_cast<unsigned>(g);
}

// Qq (int8, with sQ) when !kQ16; Qh (fp16, scales optionally to sQ_out) when kQ16.
// Vt: V_hat^T [BH][D][ld], or V_hat [BH][L][D] when kVRow.
template <int D, bool kQ16, bool kLCodes = false, bool kU8P = false, int kDbg = 0, bool kVRow = false>
int launch_attn(const int8_t *Qq, const void *Qh, const int8_t *Kq, const int8_t *Vt, const float *sQ,
                float *sQ_out, const float *sK, const float *sV, int B, int H, int L, int causal,
                void *O, cudaStream_t stream, int sshift = 0, long long cap = kWaitCycles,
                int32_t *dbg = nullptr) {
    const int BH = B * H;
    const int64_t ld = intfa_vt_ld(L);
    const CUtensorMapSwizzle swz = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap mq, mk, mv;
    int rc = make_map(&mk, Kq, D, L, BH, D, static_cast<uint64_t>(L) * D, D, BN, swz);
    if (!rc) {
        if (kQ16)   // fp16 Q rows, unswizzled (the quantiser reads them with plain loads)
            rc = make_map(&mq, Qh, D, L, BH, D * 2, static_cast<uint64_t>(L) * D * 2, D, kQHalf,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
        else
            rc = make_map(&mq, Qq, D, L, BH, D, static_cast<uint64_t>(L) * D, D, BM, swz);
    }
    if (!rc) {
        if (kVRow)   // V_hat [BH][L][D], tiles of BN rows like K_hat's
            rc = make_map(&mv, Vt, D, L, BH, D, static_cast<uint64_t>(L) * D, D, BN, swz);
        else         // V_hat^T [BH][D][ld], tiles of D rows of BN keys
            rc = make_map(&mv, Vt, ld, D, BH, ld, static_cast<uint64_t>(ld) * D, BN, D,
                          CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (rc) return rc;
    const size_t smem = attn_smem_bytes<D, kQ16>();
    auto kern = attn_fwd_kernel<D, kQ16, kLCodes, kU8P, kDbg, kVRow>;
    rc = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
    if (rc) return rc;
    // The in-kernel register split assumes exactly kLaunchRegs per thread at
    // launch; a different count could leave setmaxnreg.inc waiting forever.
    cudaFuncAttributes fa;
    rc = cuda_status(cudaFuncGetAttributes(&fa, kern));
    if (rc) return rc;
    if (fa.numRegs != kLaunchRegs) return INTFA_ERR_UNSUPPORTED;
    const int ntiles = (L + BM - 1) / BM;
    int dev = 0, nsm = 0;
    rc = cuda_status(cudaGetDevice(&dev));
    if (!rc) rc = cuda_status(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
    if (rc) return rc;
    const unsigned grid = persistent_grid(static_cast<int64_t>(BH) * ntiles, ntiles, causal, nsm);
    kern<<<grid, kThreads, smem, stream>>>(mq, mk, mv, sQ, sK, sV, static_cast<__half *>(O), BH, L, causal,
                                           static_cast<const uint4 *>(Qh), sQ_out, sshift, cap, dbg);
    return cuda_status(cudaGetLastError());
}

template <int D>
int launch_debug_qk(const int8_t *Qq, const int8_t *Kq, int BH, int L, int32_t *S,
                    cudaStream_t stream) {
    const CUtensorMapSwizzle swz = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap mq, mk;
    int rc = make_map(&mq, Qq, D, L, BH, D, static_cast<uint64_t>(L) * D, D, BM, swz);
    if (!rc) rc = make_map(&mk, Kq, D, L, BH, D, static_cast<uint64_t>(L) * D, D, BN, swz);
    if (rc) return rc;
    const size_t smem = sizeof(QKSmem<D>) + 1024;
    rc = cuda_status(cudaFuncSetAttribute(debug_qk_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(smem)));
    if (rc) return rc;
    const unsigned nt = static_cast<unsigned>((L + BM - 1) / BM);
    debug_qk_kernel<D><<<dim3(nt, nt, BH), 128, smem, stream>>>(mq, mk, L, S);
    return cuda_status(cudaGetLastError());
}

}  // namespace

int launch_attention_fwd(const int8_t *Qq, const int8_t *Kq, const int8_t *Vt, const float *sQ,
                         const float *sK, const float *sV, int B, int H, int L, int d, int causal,
                         void *O, cudaStream_t stream, int sshift) {
    if (d == 128)
        return launch_attn<128, false>(Qq, nullptr, Kq, Vt, sQ, nullptr, sK, sV, B, H, L, causal, O, stream,
                                       sshift);
    if (d == 64)
        return launch_attn<64, false>(Qq, nullptr, Kq, Vt, sQ, nullptr, sK, sV, B, H, L, causal, O, stream,
                                      sshift);
    return INTFA_ERR_UNSUPPORTED;
}

int launch_attention_fwd_vrows(const int8_t *Qq, const int8_t *Kq, const int8_t *Vq, const float *sQ,
                               const float *sK, const float *sV, int B, int H, int L, int d, int causal,
                               void *O, cudaStream_t stream) {
    if (d == 128)
        return launch_attn<128, false, false, false, 0, true>(Qq, nullptr, Kq, Vq, sQ, nullptr, sK, sV, B, H, L,
                                                              causal, O, stream);
    if (d == 64)
        return launch_attn<64, false, false, false, 0, true>(Qq, nullptr, Kq, Vq, sQ, nullptr, sK, sV, B, H, L,
                                                             causal, O, stream);
    return INTFA_ERR_UNSUPPORTED;
}

int launch_attention_debug(int mode, const int8_t *Qq, const int8_t *Kq, const int8_t *Vt, const float *sQ,
                           const float *sK, const float *sV, int B, int H, int L, int d, int causal, void *O,
                           cudaStream_t stream, long long cap, int32_t *dbg) {
    if (mode == 1) {
        if (d == 128)
            return launch_attn<128, false, false, false, 1>(Qq, nullptr, Kq, Vt, sQ, nullptr, sK, sV, B, H, L,
                                                            causal, O, stream, 0, kWaitCycles, dbg);
        return launch_attn<64, false, false, false, 1>(Qq, nullptr, Kq, Vt, sQ, nullptr, sK, sV, B, H, L, causal,
                                                       O, stream, 0, kWaitCycles, dbg);
    }
    if (mode == 2 && d == 64)
        return launch_attn<64, false, false, false, 2>(Qq, nullptr, Kq, Vt, sQ, nullptr, sK, sV, B, H, L, causal,
                                                       O, stream, 0, cap, nullptr);
    return INTFA_ERR_INVALID_ARG;
}

int launch_attention_fwd_q16(const void *Qh, const int8_t *Kq, const int8_t *Vt, const float *sK,
                             const float *sV, int B, int H, int L, int d, int causal, void *O,
                             float *sQ_out, cudaStream_t stream) {
    if (d == 128)
        return launch_attn<128, true>(nullptr, Qh, Kq, Vt, nullptr, sQ_out, sK, sV, B, H, L, causal, O, stream);
    if (d == 64)
        return launch_attn<64, true>(nullptr, Qh, Kq, Vt, nullptr, sQ_out, sK, sV, B, H, L, causal, O, stream);
    return INTFA_ERR_UNSUPPORTED;
}

}  // namespace intfa

// ------------------------------------------------------------------ C ABI ---

namespace {
int check_attn_shape(int B, int H, int L, int d) {
    if (B <= 0 || H <= 0 || L <= 0) return INTFA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return INTFA_ERR_UNSUPPORTED;
    const int64_t bh = static_cast<int64_t>(B) * H;
    if (bh > (1 << 24)) return INTFA_ERR_UNSUPPORTED;
    const int64_t tiles = (static_cast<int64_t>(L) + 127) / 128;
    if (tiles * bh > 0x7FFFFFFF) return INTFA_ERR_UNSUPPORTED;
    if (L > 131072) return INTFA_ERR_UNSUPPORTED;   // the longest sequence the tests cover
    return INTFA_OK;
}
}  // namespace

extern "C" int intfa_attention_fwd(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                                   const float *s_Q, const float *s_K, const float *s_V, int B,
                                   int H, int L, int d, int causal, void *O_f16, void *stream) {
    using namespace intfa;
    int rc = check_attn_shape(B, H, L, d);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    if (!Q_q || !K_q || !Vt_q || !s_Q || !s_K || !s_V || !O_f16) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(Q_q) || !aligned16(K_q) || !aligned16(Vt_q) || !aligned16(O_f16) ||
        (reinterpret_cast<uintptr_t>(s_Q) & 3u) || (reinterpret_cast<uintptr_t>(s_K) & 3u) ||
        (reinterpret_cast<uintptr_t>(s_V) & 3u))
        return INTFA_ERR_MISALIGNED;
    return launch_attention_fwd(Q_q, K_q, Vt_q, s_Q, s_K, s_V, B, H, L, d, causal, O_f16,
                                static_cast<cudaStream_t>(stream));
}

extern "C" int intfa_attention_fwd_vrows(const int8_t *Q_q, const int8_t *K_q, const int8_t *V_q,
                                         const float *s_Q, const float *s_K, const float *s_V, int B,
                                         int H, int L, int d, int causal, void *O_f16, void *stream) {
    using namespace intfa;
    int rc = check_attn_shape(B, H, L, d);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    if (!Q_q || !K_q || !V_q || !s_Q || !s_K || !s_V || !O_f16) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(Q_q) || !aligned16(K_q) || !aligned16(V_q) || !aligned16(O_f16) ||
        (reinterpret_cast<uintptr_t>(s_Q) & 3u) || (reinterpret_cast<uintptr_t>(s_K) & 3u) ||
        (reinterpret_cast<uintptr_t>(s_V) & 3u))
        return INTFA_ERR_MISALIGNED;
    return launch_attention_fwd_vrows(Q_q, K_q, V_q, s_Q, s_K, s_V, B, H, L, d, causal, O_f16,
                                      static_cast<cudaStream_t>(stream));
}

extern "C" int intfa_attention_fwd_blockscale(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                                              const float *s_Q, const float *s_K, const float *s_V, int B, int H,
                                              int L, int d, int causal, int scale_block, void *O_f16,
                                              void *stream) {
    using namespace intfa;
    int rc = check_attn_shape(B, H, L, d);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    int sshift = 0;
    while (sshift <= 16 && (1 << sshift) != scale_block) ++sshift;
    if (sshift > 16) return INTFA_ERR_INVALID_ARG;   // a power of two in 1 .. 65536
    if (!Q_q || !K_q || !Vt_q || !s_Q || !s_K || !s_V || !O_f16) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(Q_q) || !aligned16(K_q) || !aligned16(Vt_q) || !aligned16(O_f16) ||
        (reinterpret_cast<uintptr_t>(s_Q) & 3u) || (reinterpret_cast<uintptr_t>(s_K) & 3u) ||
        (reinterpret_cast<uintptr_t>(s_V) & 3u))
        return INTFA_ERR_MISALIGNED;
    return launch_attention_fwd(Q_q, K_q, Vt_q, s_Q, s_K, s_V, B, H, L, d, causal, O_f16,
                                static_cast<cudaStream_t>(stream), sshift);
}

extern "C" int intfa_attention_fwd_codesum(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                                           const float *s_Q, const float *s_K, const float *s_V, int B, int H,
                                           int L, int d, int causal, void *O_f16, void *stream) {
    using namespace intfa;
    int rc = check_attn_shape(B, H, L, d);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    if (!Q_q || !K_q || !Vt_q || !s_Q || !s_K || !s_V || !O_f16) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(Q_q) || !aligned16(K_q) || !aligned16(Vt_q) || !aligned16(O_f16) ||
        (reinterpret_cast<uintptr_t>(s_Q) & 3u) || (reinterpret_cast<uintptr_t>(s_K) & 3u) ||
        (reinterpret_cast<uintptr_t>(s_V) & 3u))
        return INTFA_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d == 128)
        return launch_attn<128, false, true>(Q_q, nullptr, K_q, Vt_q, s_Q, nullptr, s_K, s_V, B, H, L, causal,
                                             O_f16, s);
    return launch_attn<64, false, true>(Q_q, nullptr, K_q, Vt_q, s_Q, nullptr, s_K, s_V, B, H, L, causal, O_f16, s);
}

extern "C" int intfa_attention_fwd_pcodes(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                                          const float *s_Q, const float *s_K, const float *s_V, int B, int H,
                                          int L, int d, int causal, int p_levels, int lsum_codes, void *O_f16,
                                          void *stream) {
    using namespace intfa;
    int rc = check_attn_shape(B, H, L, d);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    if ((p_levels != 127 && p_levels != 255) || (lsum_codes != 0 && lsum_codes != 1)) return INTFA_ERR_INVALID_ARG;
    if (!Q_q || !K_q || !Vt_q || !s_Q || !s_K || !s_V || !O_f16) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(Q_q) || !aligned16(K_q) || !aligned16(Vt_q) || !aligned16(O_f16) ||
        (reinterpret_cast<uintptr_t>(s_Q) & 3u) || (reinterpret_cast<uintptr_t>(s_K) & 3u) ||
        (reinterpret_cast<uintptr_t>(s_V) & 3u))
        return INTFA_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
#define INTFA_PCODES_LAUNCH(DD, LC, U8)                                                                      \
    return launch_attn<DD, false, LC, U8>(Q_q, nullptr, K_q, Vt_q, s_Q, nullptr, s_K, s_V, B, H, L, causal, \
                                          O_f16, s)
    const bool u8 = p_levels == 255;
    if (d == 128) {
        if (u8) {
            if (lsum_codes) INTFA_PCODES_LAUNCH(128, true, true);
            INTFA_PCODES_LAUNCH(128, false, true);
        }
        if (lsum_codes) INTFA_PCODES_LAUNCH(128, true, false);
        INTFA_PCODES_LAUNCH(128, false, false);
    }
    if (u8) {
        if (lsum_codes) INTFA_PCODES_LAUNCH(64, true, true);
        INTFA_PCODES_LAUNCH(64, false, true);
    }
    if (lsum_codes) INTFA_PCODES_LAUNCH(64, true, false);
    INTFA_PCODES_LAUNCH(64, false, false);
#undef INTFA_PCODES_LAUNCH
}

extern "C" int intfa_attention_fwd_q16(const void *Q_f16, const int8_t *K_q, const int8_t *Vt_q,
                                       const float *s_K, const float *s_V, int B, int H, int L, int d,
                                       int causal, void *O_f16, float *s_Q_out, void *stream) {
    using namespace intfa;
    int rc = check_attn_shape(B, H, L, d);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    if (!Q_f16 || !K_q || !Vt_q || !s_K || !s_V || !O_f16) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(Q_f16) || !aligned16(K_q) || !aligned16(Vt_q) || !aligned16(O_f16) ||
        (reinterpret_cast<uintptr_t>(s_K) & 3u) || (reinterpret_cast<uintptr_t>(s_V) & 3u) ||
        (reinterpret_cast<uintptr_t>(s_Q_out) & 3u))
        return INTFA_ERR_MISALIGNED;
    return launch_attention_fwd_q16(Q_f16, K_q, Vt_q, s_K, s_V, B, H, L, d, causal, O_f16, s_Q_out,
                                    static_cast<cudaStream_t>(stream));
}

extern "C" int intfa_debug_qk(const int8_t *Q_q, const int8_t *K_q, int B, int H, int L, int d,
                              int32_t *S, void *stream) {
    using namespace intfa;
    int rc = check_attn_shape(B, H, L, d);
    if (rc) return rc;
    if (!Q_q || !K_q || !S) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(Q_q) || !aligned16(K_q) || !aligned16(S)) return INTFA_ERR_MISALIGNED;
    const int BH = B * H;
    if (static_cast<int64_t>((L + 127) / 128) > 65535 || BH > 65535) return INTFA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d == 128 ? launch_debug_qk<128>(Q_q, K_q, BH, L, S, s) : launch_debug_qk<64>(Q_q, K_q, BH, L, S, s);
}

extern "C" int intfa_debug_attention_scores(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                                            const float *s_Q, const float *s_K, const float *s_V, int B, int H,
                                            int L, int d, int causal, void *O_f16, int32_t *S, void *stream) {
    using namespace intfa;
    int rc = check_attn_shape(B, H, L, d);
    if (rc) return rc;
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    if (!Q_q || !K_q || !Vt_q || !s_Q || !s_K || !s_V || !O_f16 || !S) return INTFA_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * H * L * L > (int64_t{1} << 28)) return INTFA_ERR_UNSUPPORTED;
    if (!aligned16(Q_q) || !aligned16(K_q) || !aligned16(Vt_q) || !aligned16(O_f16) || !aligned16(S) ||
        (reinterpret_cast<uintptr_t>(s_Q) & 3u) || (reinterpret_cast<uintptr_t>(s_K) & 3u) ||
        (reinterpret_cast<uintptr_t>(s_V) & 3u))
        return INTFA_ERR_MISALIGNED;
    return launch_attention_debug(1, Q_q, K_q, Vt_q, s_Q, s_K, s_V, B, H, L, d, causal, O_f16,
                                  static_cast<cudaStream_t>(stream), 0, S);
}

extern "C" int intfa_debug_wait_timeout(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                                        const float *s_Q, const float *s_K, const float *s_V, int B, int H, int L,
                                        int d, int causal, void *O_f16, int64_t cap_cycles, void *stream) {
    using namespace intfa;
    int rc = check_attn_shape(B, H, L, d);
    if (rc) return rc;
    if (d != 64) return INTFA_ERR_UNSUPPORTED;
    if (causal != 0 && causal != 1) return INTFA_ERR_INVALID_ARG;
    if (cap_cycles < 1000 || cap_cycles > (int64_t{1} << 32)) return INTFA_ERR_INVALID_ARG;
    if (!Q_q || !K_q || !Vt_q || !s_Q || !s_K || !s_V || !O_f16) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(Q_q) || !aligned16(K_q) || !aligned16(Vt_q) || !aligned16(O_f16) ||
        (reinterpret_cast<uintptr_t>(s_Q) & 3u) || (reinterpret_cast<uintptr_t>(s_K) & 3u) ||
        (reinterpret_cast<uintptr_t>(s_V) & 3u))
        return INTFA_ERR_MISALIGNED;
    return launch_attention_debug(2, Q_q, K_q, Vt_q, s_Q, s_K, s_V, B, H, L, d, causal, O_f16,
                                  static_cast<cudaStream_t>(stream), static_cast<long long>(cap_cycles), nullptr);
}

extern "C" int intfa_device_status(int clear, uint32_t *word) {
    using namespace intfa;
    int rc = cuda_status(cudaDeviceSynchronize());
    if (rc) return rc;
    uint32_t w = 0, wi = 0;
    rc = cuda_status(cudaMemcpyFromSymbol(&w, g_status, sizeof(w)));
    if (rc) return rc;
    if (clear) {
        const uint32_t z = 0;
        rc = cuda_status(cudaMemcpyToSymbol(g_status, &z, sizeof(z)));
        if (rc) return rc;
    }
    rc = read_index_status(clear, &wi);   // the IndexSoftmax kernel's word
    if (rc) return rc;
    if (!w) w = wi;
    rc = read_decode_status(clear, &wi);  // the decode kernels' word
    if (rc) return rc;
    if (!w) w = wi;
    if (word) *word = w;
    return w ? INTFA_ERR_DEVICE_TIMEOUT : INTFA_OK;
}
