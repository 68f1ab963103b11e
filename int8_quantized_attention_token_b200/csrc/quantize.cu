// quantize.cu -- symmetric INT8 quantisation kernels (IntAttention: A Fully
// Integer Attention Pipeline for Efficient Edge Inference, section 2.1,
// eq. 3: s = max|x| / 127, x ~= s x_hat, zero-point 0), per token row for Q
// and K (INT-FlashAttention, abstract: token-level quantisation) and per
// L x d tensor for V.
//
// All are HBM-bound streaming kernels, one launch per tensor:
// - per token: 16 values per lane (one 32-byte load when the input is
//   32-byte aligned), warp-shuffle row maxima, 16-byte code stores;
// - per tensor: a cluster of up to 8 CTAs per group reads the group once for
//   the abs-max, combines the CTAs' maxima through distributed shared memory
//   and reads the group again, from L2, for the codes -- in the input's
//   layout, or transposed to [cols][ld] through registers.
// Two-kernel forms (abs-max, then convert) remain for the widths and the
// one-scale-for-all-groups option the cluster kernels do not take.
//
// Rounding contract (bit-exact with the definition): s = fl32(amax / 127)
// by an IEEE division; the code is RNE(fl32(x / s)) clamped to +-127.  The
// per-element quotient is formed as y = x * r with r = rcp.approx(s)
// (relative error <= 2^-23): |y - x/s| <= 127 (2^-23 + 2^-24) <= 2.3e-5 and
// |fl32(x/s) - x/s| <= 7.6e-6, so y and fl32(x/s) round to the same integer
// unless y lies within 3.1e-5 of a half-integer; when y is within 2^-14
// (6.1e-5) of one, the IEEE quotient __fdiv_rn(x, s) is used instead.  The
// result is therefore identical to rounding the IEEE quotient, at one
// multiply per element.  (A wider window costs time, not accuracy: on
// uniformly spread fractions 2^-13 of the elements take the division, so a
// 32-lane warp diverges into it on 0.4% of its element steps.)
// The scale fl32(amax / 127) is formed with Markstein's correction (P.
// Markstein, "IA-64 and Elementary Functions", 2000): q0 = amax * c with
// c = fl32(1/127), residual r = fma(-q0, 127, amax) (exact), q = fma(r, c, q0).
// amax is always an fp16 magnitude; the GPU tests check q against the IEEE
// quotient for every finite fp16 value.
// RNE itself is fl(y + 1.5 * 2^23): for |y| < 2^22 that float is
// 1.5 * 2^23 + RNE(y) exactly, so its low byte is the code in two's complement
// and y - (t - 1.5 * 2^23) is the exact rounding residual.  |fl32(x/s)| never
// exceeds 127.00002, so the +-127 clamp never binds.
#include <cuda_fp16.h>

#include <mutex>

#include "internal.h"
#include "quant_math.cuh"

namespace intfa {
namespace {

using namespace qmath;

// ------------------------------------------------------------ per token ---

// G lanes cover one row of d = 8 G values; a warp holds 32 / G rows per
// slice and strides over the rows by the whole grid.  Each thread issues the
// 16-byte load of its next slice before the arithmetic on the current one, so
// two loads per thread are in flight (six 256-thread blocks per SM).
template <int G>
__global__ void __launch_bounds__(256, 6) quant_per_token_kernel(const uint4 *__restrict__ x,
                                                                 int64_t rows,
                                                                 uint2 *__restrict__ xq,
                                                                 float *__restrict__ scale) {
    const int lane = threadIdx.x & 31;
    const int sub = lane & (G - 1);
    constexpr int kRowsPerWarp = 32 / G;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t step = nwarps * kRowsPerWarp;
    int64_t r = warp * kRowsPerWarp + lane / G;
    uint4 v = r < rows ? __ldcs(x + r * G + sub) : make_uint4(0u, 0u, 0u, 0u);
    for (int64_t r0 = warp * kRowsPerWarp; r0 < rows; r0 += step) {
        const int64_t rn = r + step;
        const uint4 vn = rn < rows ? __ldcs(x + rn * G + sub) : make_uint4(0u, 0u, 0u, 0u);
        float f[8];
        unpack8(v, f);
        float amax = absmax8(f);
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        const float s = div127(amax);
        const float rcp = rcp_or_zero(s);
        if (r < rows) {
            __stcs(xq + r * G + sub, codes8(f, s, rcp));
            if (sub == 0) scale[r] = s;
        }
        r = rn;
        v = vn;
    }
}

// ----------------------------------------------------------- per tensor ---

// Phase 1: max |x| per group into ws[g] (fp32 bit pattern; atomicMax on the
// unsigned bits orders non-negative floats correctly).  ws zeroed before.
__global__ void __launch_bounds__(256) group_amax_kernel(const uint4 *__restrict__ x,
                                                         int64_t n8, unsigned *__restrict__ ws) {
    const int g = blockIdx.y;
    const uint4 *xg = x + static_cast<int64_t>(g) * n8;
    float m = 0.0f;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float f[8];
        unpack8(__ldg(xg + i), f);
        m = fmaxf(m, absmax8(f));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ float part[8];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (blockDim.x >> 5); ++w) m = fmaxf(m, part[w]);
        atomicMax(ws + g, __float_as_uint(m));
    }
}

// Between the phases, for one scale over all groups: every group's slot gets
// the maximum over the groups (one block).
__global__ void __launch_bounds__(256) global_amax_kernel(unsigned *__restrict__ ws, int64_t groups) {
    unsigned m = 0u;
    for (int64_t g = threadIdx.x; g < groups; g += blockDim.x) m = max(m, ws[g]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ unsigned part[8];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
    __syncthreads();
    m = part[0];
    for (int w = 1; w < (blockDim.x >> 5); ++w) m = max(m, part[w]);
    for (int64_t g = threadIdx.x; g < groups; g += blockDim.x) ws[g] = m;
}

// Phase 2, same layout as the input.
__global__ void __launch_bounds__(256) group_convert_kernel(const uint4 *__restrict__ x,
                                                            int64_t n8,
                                                            const unsigned *__restrict__ ws,
                                                            uint2 *__restrict__ xq,
                                                            float *__restrict__ scale) {
    const int g = blockIdx.y;
    const float s = div127(__uint_as_float(ws[g]));
    const float rcp = rcp_or_zero(s);
    if (blockIdx.x == 0 && threadIdx.x == 0) scale[g] = s;
    const uint4 *xg = x + static_cast<int64_t>(g) * n8;
    uint2 *qg = xq + static_cast<int64_t>(g) * n8;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float f[8];
        unpack8(__ldcs(xg + i), f);
        __stcs(qg + i, codes8(f, s, rcp));
    }
}

// Phase 2, transposed: group g of [rows][cols] -> [cols][ld]; rows in
// [rows, ld) get code 0.  A block covers kTRG row groups of 4 rows: thread
// (rg, c8) loads rows 4 rg .. 4 rg + 3 of columns 8 c8 .. 8 c8 + 7 (16-byte
// coalesced loads), packs the 4 codes of each column into one 32-bit word and
// stores the 8 words to shared memory, column-major with a one-word pad and a
// per-thread rotation of the column order (bank-conflict-light); the block then
// writes each column's 4 kTRG bytes with 16-byte stores.
constexpr int kTRG = 16;              // row groups of 4 per block (64 rows)
constexpr int kTRows = 4 * kTRG;
__global__ void __launch_bounds__(256, 6) group_convert_t_kernel(const uint4 *__restrict__ x,
                                                              int64_t rows, int cols, int64_t ld,
                                                              const unsigned *__restrict__ ws,
                                                              int8_t *__restrict__ xq,
                                                              float *__restrict__ scale) {
    __shared__ uint32_t tile[256 * (kTRG + 1)];   // [col][row group], padded
    const int g = blockIdx.y;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kTRows;
    const float s = div127(__uint_as_float(ws[g]));
    const float rcp = rcp_or_zero(s);
    if (blockIdx.x == 0 && threadIdx.x == 0) scale[g] = s;
    const int c8n = cols >> 3;
    const uint4 *xg = x + static_cast<int64_t>(g) * rows * c8n;
    for (int t = threadIdx.x; t < kTRG * c8n; t += blockDim.x) {
        const int c8 = t % c8n, rg = t / c8n;
        uint2 w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int64_t r = r0 + 4 * rg + k;
            w[k] = make_uint2(0u, 0u);
            if (r < rows) {
                float f[8];
                unpack8(__ldcs(xg + r * c8n + c8), f);
                w[k] = codes8(f, s, rcp);
            }
        }
        // column e's word = byte e of rows 0..3 (PRMT selects byte e of
        // the first and byte e of the second source, then interleaves)
        uint32_t col[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t sel = static_cast<uint32_t>(e | ((e + 4) << 4));
            col[e] = prmt(prmt(w[0].x, w[1].x, sel), prmt(w[2].x, w[3].x, sel), 0x5410u);
            col[e + 4] = prmt(prmt(w[0].y, w[1].y, sel), prmt(w[2].y, w[3].y, sel), 0x5410u);
        }
        const int rot = (c8 >> 2) & 7;
#pragma unroll
        for (int e0 = 0; e0 < 8; ++e0) {
            const int e = (e0 + rot) & 7;
            tile[(8 * c8 + e) * (kTRG + 1) + rg] = col[e];
        }
    }
    __syncthreads();
    int8_t *qg = xq + static_cast<int64_t>(g) * cols * ld;
    for (int j = threadIdx.x; j < cols * (kTRG / 4); j += blockDim.x) {
        const int c = j / (kTRG / 4), part = j % (kTRG / 4);
        const int64_t rr = r0 + 16 * part;
        if (rr < ld) {
            const uint32_t *src = &tile[c * (kTRG + 1) + 4 * part];
            __stcs(reinterpret_cast<uint4 *>(qg + c * ld + rr), make_uint4(src[0], src[1], src[2], src[3]));
        }
    }
}

// Phase 2, transposed, persistent form: each block walks tiles of 128 rows
// of one group (tile k, k + grid, ...), so that every column of a tile is a
// full 128-byte run of the output; while the current tile's columns are
// written, the next tile's rows are already being loaded.  Thread tasks are
// (row group of 4 rows, 8 columns) pairs as in group_convert_t_kernel.
constexpr int kPRows = 128;                 // rows per tile
constexpr int kPRG = kPRows / 4;            // row groups per tile
constexpr int kPThreads = 256;
template <int C8>                           // columns / 8 (cols <= 256)
__global__ void __launch_bounds__(kPThreads, 4) group_convert_tp_kernel(const uint4 *__restrict__ x,
                                                                        int64_t rows, int64_t ld, int64_t groups,
                                                                        const unsigned *__restrict__ ws,
                                                                        int8_t *__restrict__ xq,
                                                                        float *__restrict__ scale) {
    constexpr int kCols = 8 * C8;
    constexpr int kTasks = kPRG * C8;                           // (row group, 8 columns) pairs per tile
    constexpr int kPer = (kTasks + kPThreads - 1) / kPThreads;  // tasks per thread
    __shared__ uint32_t tile[kCols * (kPRG + 1)];               // [col][row group], padded
    const int64_t ntile = (ld + kPRows - 1) / kPRows;
    const int64_t total = groups * ntile;
    int64_t T = blockIdx.x;
    uint4 buf[kPer][4];
    // loads of tile T's rows for this thread's tasks (zeros past the end)
    auto load = [&](int64_t tt) {
        const int64_t g = tt / ntile, r0 = (tt - g * ntile) * kPRows;
        const uint4 *xg = x + g * rows * C8;
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int t = threadIdx.x + q * kPThreads;
            const int c8 = t % C8, rg = t / C8;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int64_t r = r0 + 4 * rg + k;
                buf[q][k] = (t < kTasks && r < rows) ? __ldcs(xg + r * C8 + c8) : make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    if (T < total) load(T);
    for (; T < total; T += gridDim.x) {
        const int64_t g = T / ntile, r0 = (T - g * ntile) * kPRows;
        const float s = div127(__uint_as_float(ws[g]));
        const float rcp = rcp_or_zero(s);
        if (r0 == 0 && threadIdx.x == 0) scale[g] = s;
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int t = threadIdx.x + q * kPThreads;
            if (t >= kTasks) continue;
            const int c8 = t % C8, rg = t / C8;
            uint2 w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float f[8];
                unpack8(buf[q][k], f);
                w[k] = codes8(f, s, rcp);   // rows past the end were loaded as zeros: code 0
            }
            uint32_t col[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t sel = static_cast<uint32_t>(e | ((e + 4) << 4));
                col[e] = prmt(prmt(w[0].x, w[1].x, sel), prmt(w[2].x, w[3].x, sel), 0x5410u);
                col[e + 4] = prmt(prmt(w[0].y, w[1].y, sel), prmt(w[2].y, w[3].y, sel), 0x5410u);
            }
            const int rot = (c8 >> 2) & 7;
#pragma unroll
            for (int e0 = 0; e0 < 8; ++e0) {
                const int e = (e0 + rot) & 7;
                tile[(8 * c8 + e) * (kPRG + 1) + rg] = col[e];
            }
        }
        __syncthreads();
        // the next tile's loads go out before this tile's stores
        if (T + gridDim.x < total) load(T + gridDim.x);
        int8_t *qg = xq + g * kCols * ld;
        for (int j = threadIdx.x; j < kCols * (kPRG / 4); j += kPThreads) {
            const int c = j / (kPRG / 4), part = j % (kPRG / 4);
            const int64_t rr = r0 + 16 * part;
            if (rr < ld) {
                const uint32_t *src = &tile[c * (kPRG + 1) + 4 * part];
                __stcs(reinterpret_cast<uint4 *>(qg + c * ld + rr), make_uint4(src[0], src[1], src[2], src[3]));
            }
        }
        __syncthreads();
    }
}

// Both phases of the per-tensor quantiser with the transposed output in one
// kernel: a cluster of CL CTAs per group.  Each CTA takes the group's tiles
// of 128 rows k, k + CL, ... ; it reads them once for the abs-max, the CL
// partial maxima are combined through distributed shared memory (cluster
// barrier, remote shared-memory loads), and each CTA then reads its tiles
// again -- from L2, where the first pass has just put them with an
// evict-last hint -- to write the transposed codes.  HBM sees 2 bytes read
// and 1 written per element, against 4 and 1 for the two-kernel path.  The
// maximum is order-independent, so s and the codes equal the two-kernel
// path's bit for bit.
//
// The second pass needs no shared memory: lane l of a warp holds rows
// 4l .. 4l + 3 of a 128-row tile for 16 columns (one 32-byte load per row),
// packs the 4 codes of each column into one word, and the warp's 32 words of
// a column are one contiguous 128-byte run of the output.  The per-element
// arithmetic is 1 conversion, 1.5 packed FMAs and a shared near-tie test
// per 8 elements (see code_cols below), which keeps the kernel memory-bound.
constexpr int kCL = 8;                      // CTAs per group (cluster size), at least
constexpr int kCLMax = 16;                  //   ... and at most (a non-portable size)
// CTAs per cluster for `groups` groups of `units` work units (row tiles or
// blocks) each: 8, raised toward 16 when there are few groups so that about
// 512 CTAs (four per SM) run; never more than the units.  (32 heads of
// 16384 x 128: 105 us with 8, 76 us with 16; 128 heads of 4096 x 128: 59 us
// either way.)
int cluster_ctas(int64_t groups, int64_t units) {
    int64_t want = (512 + groups - 1) / groups;
    want = want < kCL ? kCL : (want > kCLMax ? kCLMax : want);
    return static_cast<int>(units < want ? units : want);
}
// Launches `kernel` (kPThreads threads per CTA) as `groups` clusters of `cl`
// CTAs on `stream`.  A size above kCL is non-portable: the kernel is allowed
// it first (on the current device, at every such launch), and a device that
// cannot schedule it gets the portable size kCL instead -- the kernels read
// their cluster size at run time.
template <typename... KArgs, typename... Args>
int launch_clusters(void (*kernel)(KArgs...), int64_t groups, int cl, cudaStream_t stream, Args... args) {
    for (;;) {
        if (cl > kCL) {
            const int rc = cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
            if (rc) return rc;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(groups * cl), 1, 1);
        cfg.blockDim = dim3(kPThreads, 1, 1);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(cl);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
        if (e == cudaSuccess) return INTFA_OK;
        if (cl <= kCL) return cuda_status(e);
        (void)cudaGetLastError();   // not sticky: retry with the portable size
        cl = kCL;
    }
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(const float *local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// Read-only loads with an L2 eviction-priority hint: the first pass marks a
// group's rows evict-last so that they are still in L2 when the second pass
// reads them (evict-first there: nothing reads them after that).
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint4 ld_hint(const uint4 *p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}
// 32 bytes (16 fp16 values) from a 32-byte aligned address.
__device__ __forceinline__ void ld32_hint(const uint4 *p, uint64_t pol, uint32_t (&w)[8]) {
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8], %9;"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p), "l"(pol));
}

// The codes of a 4-row x 2-column block, one word per column: wk[k] holds
// the fp16 pair (column 0, column 1) of row k; c0 / c1 get the codes of
// column 0 / 1 for rows 0..3 in bytes 0..3.  Same contract as code_bits:
// t = fl(x r + 1.5 2^23) is 1.5 2^23 + RNE(x r) (|x r| <= 127.0001), and
// x r differs from x / s by at most 127 * 2^-23, fl32(x / s) from x / s by at
// most 7.6e-6, so RNE(x r) is the contract's code unless x r lies within
// 2.3e-5 of a half-integer.  The rounding residual x r - RNE(x r) is
// fma(x, r, 1.5 2^23 - t) (1.5 2^23 - t is exact, the fma adds at most
// 3e-8); when any of the 8 lies beyond kNearTie = 0.5 - 2^-14 in magnitude,
// those elements take the IEEE quotient.
__device__ __forceinline__ void code_cols(const uint32_t (&wk)[4], float s, float r, uint32_t &c0, uint32_t &c1) {
    const uint64_t r2 = f2_pack(r, r), k2 = f2_pack(kRound, kRound), m2 = f2_pack(-1.0f, -1.0f);
    uint32_t t0[4], t1[4];
    float worst = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&wk[k]));
        const uint64_t x2 = f2_pack(f.x, f.y);
        const uint64_t t2 = ffma2(x2, r2, k2);
        const uint64_t e2 = ffma2(x2, r2, ffma2(t2, m2, k2));
        float a, b, ea, eb;
        f2_unpack(t2, a, b);
        f2_unpack(e2, ea, eb);
        t0[k] = __float_as_uint(a);
        t1[k] = __float_as_uint(b);
        worst = fmaxf(worst, fmaxf(fabsf(ea), fabsf(eb)));
    }
    if (worst > kNearTie) {   // a near-tie: the IEEE quotient for those elements
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&wk[k]));
            const float ta = fmaf(f.x, r, kRound), tb = fmaf(f.y, r, kRound);
            if (fabsf(fmaf(f.x, r, kRound - ta)) > kNearTie) t0[k] = __float_as_uint(__fdiv_rn(f.x, s) + kRound);
            if (fabsf(fmaf(f.y, r, kRound - tb)) > kNearTie) t1[k] = __float_as_uint(__fdiv_rn(f.y, s) + kRound);
        }
    }
    c0 = prmt(prmt(t0[0], t0[1], 0x0040u), prmt(t0[2], t0[3], 0x0040u), 0x5410u);
    c1 = prmt(prmt(t1[0], t1[1], 0x0040u), prmt(t1[2], t1[3], 0x0040u), 0x5410u);
}

// The codes of 16 consecutive values (w: 8 fp16 pairs), packed little-endian
// into 16 bytes; same arithmetic and near-tie rule as code_cols, one test per
// 16 values.
__device__ __forceinline__ uint4 codes16(const uint32_t (&w)[8], float s, float r) {
    const uint64_t r2 = f2_pack(r, r), k2 = f2_pack(kRound, kRound), m2 = f2_pack(-1.0f, -1.0f);
    uint32_t q[4];
    float worst = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {   // output word i: values 4i .. 4i + 3 (pairs w[2i], w[2i + 1])
        uint32_t t[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[2 * i + h]));
            const uint64_t x2 = f2_pack(f.x, f.y);
            const uint64_t t2 = ffma2(x2, r2, k2);
            const uint64_t e2 = ffma2(x2, r2, ffma2(t2, m2, k2));
            float a, b, ea, eb;
            f2_unpack(t2, a, b);
            f2_unpack(e2, ea, eb);
            t[2 * h] = __float_as_uint(a);
            t[2 * h + 1] = __float_as_uint(b);
            worst = fmaxf(worst, fmaxf(fabsf(ea), fabsf(eb)));
        }
        q[i] = prmt(prmt(t[0], t[1], 0x0040u), prmt(t[2], t[3], 0x0040u), 0x5410u);
    }
    if (worst > kNearTie) {   // a near-tie: redo the 16 codes, the IEEE quotient where needed
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t t[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[2 * i + h]));
                const float ta = fmaf(f.x, r, kRound), tb = fmaf(f.y, r, kRound);
                t[2 * h] = __float_as_uint(fabsf(fmaf(f.x, r, kRound - ta)) > kNearTie ? __fdiv_rn(f.x, s) + kRound : ta);
                t[2 * h + 1] = __float_as_uint(fabsf(fmaf(f.y, r, kRound - tb)) > kNearTie ? __fdiv_rn(f.y, s) + kRound : tb);
            }
            q[i] = prmt(prmt(t[0], t[1], 0x0040u), prmt(t[2], t[3], 0x0040u), 0x5410u);
        }
    }
    return make_uint4(q[0], q[1], q[2], q[3]);
}

// 16 fp16 values (32 bytes) at p: one 32-byte load when kV8 (p 32-byte
// aligned), else two 16-byte loads.
template <bool kV8>
__device__ __forceinline__ void ld16v(const uint4 *p, uint64_t pol, uint32_t (&w)[8]) {
    if constexpr (kV8) {
        ld32_hint(p, pol, w);
    } else {
        const uint4 a = ld_hint(p, pol), b = ld_hint(p + 1, pol);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
}

// Exact abs-max of 16 fp16 values, as fp16 bits (non-negative fp16 values
// order like their bit patterns).
__device__ __forceinline__ uint32_t absmax16_bits(const uint32_t (&w)[8]) {
    __half2 m = __habs2(*reinterpret_cast<const __half2 *>(&w[0]));
#pragma unroll
    for (int i = 1; i < 8; ++i) m = __hmax2(m, __habs2(*reinterpret_cast<const __half2 *>(&w[i])));
    return __half_as_ushort(__hmax(__low2half(m), __high2half(m)));
}

// Per token, 16 values per lane: G = d / 16 lanes cover a row, a warp holds
// 32 / G rows per step and strides over the rows by the whole grid; the next
// step's loads are issued before the current step's arithmetic.  The row
// maximum is reduced on fp16 bit patterns, the codes use codes16.
template <int G, bool kV8>
__global__ void __launch_bounds__(256, 4) quant_per_token16_kernel(const uint4 *__restrict__ x, int64_t rows,
                                                                   uint4 *__restrict__ xq,
                                                                   float *__restrict__ scale) {
    const int lane = threadIdx.x & 31;
    const int sub = lane & (G - 1);
    constexpr int kRowsPerWarp = 32 / G;
    const uint64_t pol = l2_policy_evict_first();
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t step = nwarps * kRowsPerWarp;
    int64_t r = warp * kRowsPerWarp + lane / G;
    uint32_t v[8];
    auto load = [&](int64_t row, uint32_t (&w)[8]) {
        if (row < rows) {
            ld16v<kV8>(x + (row * G + sub) * 2, pol, w);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = 0u;
        }
    };
    load(r, v);
    for (int64_t r0 = warp * kRowsPerWarp; r0 < rows; r0 += step) {
        const int64_t rn = r + step;
        uint32_t vn[8];
        load(rn, vn);
        uint32_t mb = absmax16_bits(v);
#pragma unroll
        for (int o = G / 2; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
        const float s = div127(__half2float(__ushort_as_half(static_cast<unsigned short>(mb))));
        const float rcp = rcp_or_zero(s);
        const uint4 q = codes16(v, s, rcp);
        if (r < rows) {
            __stcs(xq + r * G + sub, q);
            if (sub == 0) scale[r] = s;
        }
        r = rn;
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = vn[i];
    }
}

// Per-tensor quantiser, codes in the input's layout, both phases in one
// kernel: a cluster of CL CTAs per group as in the transposed form.  A group
// is n16 runs of 16 values; CTA k of the cluster takes the blocks of 256 runs
// k, k + CL, ...  (one run per thread and block), reads them for the abs-max
// (evict-last), and after the cluster-wide maximum reads them again, last
// block first, to write the codes (one 16-byte store per run).
template <bool kV8>
__global__ void __launch_bounds__(kPThreads, 4) group_quant_fused_kernel(const uint4 *__restrict__ x,
                                                                         int64_t n16,
                                                                         uint4 *__restrict__ xq,
                                                                         float *__restrict__ scale) {
    constexpr int kWarps = kPThreads / 32;
    constexpr int kU = 4;                                   // runs in flight per thread
    __shared__ uint32_t part[kWarps];
    __shared__ float cmax;
    const uint32_t rank = cluster_rank(), ncl = cluster_size();
    const int64_t g = blockIdx.x / ncl;
    const int64_t nblk = (n16 + kPThreads - 1) / kPThreads;
    const int64_t mine = (nblk - 1 - rank) / ncl + 1;      // blocks of this CTA (rank < nblk)
    const uint4 *xg = x + g * n16 * 2;
    uint4 *qg = xq + g * n16;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();
    auto run = [&](int64_t i) { return (rank + i * ncl) * kPThreads + threadIdx.x; };   // i-th block's run
    uint32_t mb = 0u;
    for (int64_t i0 = 0; i0 < mine; i0 += kU) {
        uint32_t w[kU][8];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t c = run(i0 + u);
            if (i0 + u < mine && c < n16) {
                ld16v<kV8>(xg + 2 * c, keep, w[u]);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) w[u][k] = 0u;
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) mb = max(mb, absmax16_bits(w[u]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
    if (lane == 0) part[warp] = mb;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < kWarps; ++i) mb = max(mb, part[i]);
        cmax = __half2float(__ushort_as_half(static_cast<unsigned short>(mb)));
    }
    cluster_sync_all();   // every CTA's cmax is written and visible
    float amax = 0.0f;
    for (uint32_t i = 0; i < ncl; ++i) amax = fmaxf(amax, ld_cluster_f32(&cmax, i));
    cluster_arrive();     // this CTA has read every cmax (waited for at the end)
    const float s = div127(amax);
    const float rcp = rcp_or_zero(s);
    if (rank == 0 && threadIdx.x == 0) scale[g] = s;
    for (int64_t i0 = mine - 1; i0 >= 0; i0 -= 2) {
        uint32_t w[2][8];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t c = run(i0 - u);
            if (i0 - u >= 0 && c < n16) {
                ld16v<kV8>(xg + 2 * c, drop, w[u]);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) w[u][k] = 0u;
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t c = run(i0 - u);
            const uint4 q = codes16(w[u], s, rcp);
            if (i0 - u >= 0 && c < n16) __stcs(qg + c, q);
        }
    }
    cluster_wait();       // no CTA leaves while another may still read its cmax
}

int launch_quant_fused(const uint4 *x, int64_t groups, int64_t n16, int8_t *xq, float *scale,
                       cudaStream_t stream) {
    const int64_t nblk = (n16 + kPThreads - 1) / kPThreads;
    const int cl = cluster_ctas(groups, nblk);
    uint4 *q = reinterpret_cast<uint4 *>(xq);
    if ((reinterpret_cast<uintptr_t>(x) & 31u) == 0)
        return launch_clusters(group_quant_fused_kernel<true>, groups, cl, stream, x, n16, q, scale);
    return launch_clusters(group_quant_fused_kernel<false>, groups, cl, stream, x, n16, q, scale);
}

template <int C8, bool kV8>     // kV8: the input is 32-byte aligned (one load per row)
__global__ void __launch_bounds__(kPThreads, 4) group_quant_t_fused_kernel(const uint4 *__restrict__ x,
                                                                           int64_t rows, int64_t ld,
                                                                           int8_t *__restrict__ xq,
                                                                           float *__restrict__ scale) {
    static_assert(C8 % 2 == 0 && kPRows * C8 % kPThreads == 0, "tile shape");
    constexpr int kCB = C8 / 2;                             // 16-column blocks per tile
    constexpr int kWarps = kPThreads / 32;
    __shared__ float part[kWarps];
    __shared__ float cmax;                   // this CTA's abs-max, read by the cluster
    const uint32_t rank = cluster_rank(), ncl = cluster_size();
    const int64_t g = blockIdx.x / ncl;
    const int64_t ntile = (ld + kPRows - 1) / kPRows;
    const int64_t mine = (ntile - 1 - rank) / ncl + 1;     // tiles of this CTA (rank < ntile)
    const uint4 *xg = x + g * rows * C8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();
    // -- pass 1: abs-max over this CTA's tiles, coalesced 16-byte loads,
    // packed fp16 maxima (exact: fp16 magnitudes order like their fp32 values)
    constexpr int kLd = kPRows * C8 / kPThreads;           // 16-byte loads per thread per tile
    constexpr int kU = kLd < 8 ? kLd : 8;                   // issued together, then reduced
    __half2 m2 = __float2half2_rn(0.0f);
    for (int64_t T = rank; T < ntile; T += ncl) {
        const int64_t r0 = T * kPRows;
#pragma unroll
        for (int u0 = 0; u0 < kLd; u0 += kU) {
            uint4 v[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int t = threadIdx.x + (u0 + u) * kPThreads;
                const int64_t r = r0 + t / C8;
                v[u] = r < rows ? ld_hint(xg + r * C8 + t % C8, keep) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const __half2 *h = reinterpret_cast<const __half2 *>(&v[u]);
#pragma unroll
                for (int i = 0; i < 4; ++i) m2 = __hmax2(m2, __habs2(h[i]));
            }
        }
    }
    // -- pass 2 tasks: (tile, 16-column block), this CTA's tiles last first
    // (the most recently read rows are the likeliest still in L2); warp w
    // takes tasks w, w + 8, ...; the first task's loads go out before the
    // cluster barrier
    const int64_t ntask = mine * kCB;
    uint32_t w[4][8];
    auto load = [&](int64_t task) {
        const int64_t T = rank + (mine - 1 - task / kCB) * ncl;
        const int cb = static_cast<int>(task % kCB);
        const int64_t r = T * kPRows + 4 * lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (r + k < rows) {
                const uint4 *p = xg + (r + k) * C8 + 2 * cb;
                if constexpr (kV8) {
                    ld32_hint(p, drop, w[k]);
                } else {
                    const uint4 a = ld_hint(p, drop), b = ld_hint(p + 1, drop);
                    w[k][0] = a.x; w[k][1] = a.y; w[k][2] = a.z; w[k][3] = a.w;
                    w[k][4] = b.x; w[k][5] = b.y; w[k][6] = b.z; w[k][7] = b.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) w[k][i] = 0u;
            }
        }
    };
    if (warp < ntask) load(warp);
    float m = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) part[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < kWarps; ++i) m = fmaxf(m, part[i]);
        cmax = m;
    }
    cluster_sync_all();   // every CTA's cmax is written and visible
    float amax = 0.0f;
    for (uint32_t i = 0; i < ncl; ++i) amax = fmaxf(amax, ld_cluster_f32(&cmax, i));
    cluster_arrive();     // this CTA has read every cmax (waited for at the end)
    const float s = div127(amax);
    const float rcp = rcp_or_zero(s);
    if (rank == 0 && threadIdx.x == 0) scale[g] = s;
    int8_t *qg = xq + g * (8 * C8) * ld;
    for (int64_t task = warp; task < ntask; task += kWarps) {
        if (task != warp) load(task);
        const int64_t T = rank + (mine - 1 - task / kCB) * ncl;
        const int cb = static_cast<int>(task % kCB);
        const int64_t r = T * kPRows + 4 * lane;
        uint32_t *out = reinterpret_cast<uint32_t *>(qg + (16 * cb) * ld + r);
#pragma unroll
        for (int p = 0; p < 8; ++p) {       // columns 16 cb + 2p, 16 cb + 2p + 1
            const uint32_t wk[4] = {w[0][p], w[1][p], w[2][p], w[3][p]};
            uint32_t c0, c1;
            code_cols(wk, s, rcp, c0, c1);
            if (r < ld) {                   // rows in [rows, ld) were loaded as zeros: code 0
                __stcs(out + (2 * p) * (ld / 4), c0);
                __stcs(out + (2 * p + 1) * (ld / 4), c1);
            }
        }
    }
    cluster_wait();       // no CTA leaves while another may still read its cmax
}

template <int C8>
int launch_quant_t_fused(const uint4 *x, int64_t groups, int64_t rows, int64_t ld, int8_t *xq, float *scale,
                         cudaStream_t stream) {
    const int64_t ntile = (ld + kPRows - 1) / kPRows;
    const int cl = cluster_ctas(groups, ntile);
    if ((reinterpret_cast<uintptr_t>(x) & 31u) == 0)
        return launch_clusters(group_quant_t_fused_kernel<C8, true>, groups, cl, stream, x, rows, ld, xq, scale);
    return launch_clusters(group_quant_t_fused_kernel<C8, false>, groups, cl, stream, x, rows, ld, xq, scale);
}

int grid_for(int64_t work_items, int per_block) {
    int64_t blocks = (work_items + per_block - 1) / per_block;
    const int64_t cap = 148 * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return static_cast<int>(blocks);
}

}  // namespace

// b-bit symmetric codes, one scale per row: s = fl(max|x| / qmax) and
// code = clamp(RNE(x / s), -qmax, qmax), both IEEE divisions (a variant for
// narrow codes, not on the INT8 hot path).  G lanes per row of 8 G values.
template <int G>
__global__ void __launch_bounds__(256) quant_per_token_bits_kernel(const uint4 *__restrict__ x, int64_t rows,
                                                                 float qmax, uint2 *__restrict__ xq,
                                                                 float *__restrict__ scale) {
    const int sub = threadIdx.x % G;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / G) + threadIdx.x / G;
    const bool live = row < rows;
    float f[8];
    float amax = 0.0f;
    if (live) {
        unpack8(__ldg(x + row * G + sub), f);
        amax = absmax8(f);
    }
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (!live) return;
    const float s = __fdiv_rn(amax, qmax);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        int c = 0;
        if (s != 0.0f) c = max(-static_cast<int>(qmax), min(static_cast<int>(qmax), __float2int_rn(__fdiv_rn(f[e], s))));
        w[e >> 2] |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * (e & 3));
    }
    xq[row * G + sub] = make_uint2(w[0], w[1]);
    if (sub == 0) scale[row] = s;
}

int launch_quantize_per_token_bits(const void *x, int64_t rows, int d, int bits, int8_t *xq, float *scale,
                                   cudaStream_t stream) {
    if (rows == 0) return INTFA_OK;
    const uint4 *xv = static_cast<const uint4 *>(x);
    uint2 *qv = reinterpret_cast<uint2 *>(xq);
    const float qmax = static_cast<float>((1 << (bits - 1)) - 1);
    const int grid = grid_for(rows, 256 / (d / 8));
    switch (d) {
        case 8: quant_per_token_bits_kernel<1><<<grid, 256, 0, stream>>>(xv, rows, qmax, qv, scale); break;
        case 16: quant_per_token_bits_kernel<2><<<grid, 256, 0, stream>>>(xv, rows, qmax, qv, scale); break;
        case 32: quant_per_token_bits_kernel<4><<<grid, 256, 0, stream>>>(xv, rows, qmax, qv, scale); break;
        case 64: quant_per_token_bits_kernel<8><<<grid, 256, 0, stream>>>(xv, rows, qmax, qv, scale); break;
        case 128: quant_per_token_bits_kernel<16><<<grid, 256, 0, stream>>>(xv, rows, qmax, qv, scale); break;
        case 256: quant_per_token_bits_kernel<32><<<grid, 256, 0, stream>>>(xv, rows, qmax, qv, scale); break;
        default: return INTFA_ERR_UNSUPPORTED;
    }
    return cuda_status(cudaGetLastError());
}

int launch_quantize_per_token(const void *x, int64_t rows, int d, int8_t *xq, float *scale,
                              cudaStream_t stream) {
    if (rows == 0) return INTFA_OK;
    const uint4 *xv = static_cast<const uint4 *>(x);
    if (d == 8) {   // one lane per row, 8 values
        quant_per_token_kernel<1><<<grid_for(rows, 256), 256, 0, stream>>>(xv, rows, reinterpret_cast<uint2 *>(xq),
                                                                          scale);
        return cuda_status(cudaGetLastError());
    }
    // 16 values per lane; one 32-byte load per lane when x is 32-byte aligned
    uint4 *qv = reinterpret_cast<uint4 *>(xq);
    const int grid = grid_for(rows, 256 / (d / 16));
    const bool v8 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0;
#define INTFA_PT16(G)                                                                     \
    (v8 ? quant_per_token16_kernel<G, true><<<grid, 256, 0, stream>>>(xv, rows, qv, scale) \
        : quant_per_token16_kernel<G, false><<<grid, 256, 0, stream>>>(xv, rows, qv, scale))
    switch (d) {
        case 16: INTFA_PT16(1); break;
        case 32: INTFA_PT16(2); break;
        case 64: INTFA_PT16(4); break;
        case 128: INTFA_PT16(8); break;
        case 256: INTFA_PT16(16); break;
        default: return INTFA_ERR_UNSUPPORTED;
    }
#undef INTFA_PT16
    return cuda_status(cudaGetLastError());
}

int launch_quantize_per_tensor(const void *x, int64_t groups, int64_t rows, int cols,
                               int transpose, int8_t *xq, float *scale, void *workspace,
                               cudaStream_t stream, bool global) {
    if (groups == 0) return INTFA_OK;
    if (!transpose && !global && cols % 16 == 0 && groups <= (int64_t(1) << 24))
        return launch_quant_fused(static_cast<const uint4 *>(x), groups, rows * cols / 16, xq, scale, stream);
    if (transpose && !global && groups <= (int64_t(1) << 24)) {
        // one kernel: a cluster per group, abs-max and transposed codes
        const int64_t ld = intfa_vt_ld(rows);
        const uint4 *xv = static_cast<const uint4 *>(x);
        switch (cols / 8) {
            case 4: return launch_quant_t_fused<4>(xv, groups, rows, ld, xq, scale, stream);
            case 8: return launch_quant_t_fused<8>(xv, groups, rows, ld, xq, scale, stream);
            case 16: return launch_quant_t_fused<16>(xv, groups, rows, ld, xq, scale, stream);
            default: break;   // other widths: the two-kernel path below
        }
    }
    unsigned *ws = static_cast<unsigned *>(workspace);
    int rc = cuda_status(cudaMemsetAsync(ws, 0, static_cast<size_t>(groups) * sizeof(unsigned), stream));
    if (rc) return rc;
    const int64_t n8 = rows * cols / 8;
    const uint4 *xv = static_cast<const uint4 *>(x);
    int chunks = static_cast<int>((148 * 8 + groups - 1) / groups);
    const int64_t max_chunks = (n8 + 255) / 256;
    if (chunks > max_chunks) chunks = static_cast<int>(max_chunks);
    if (chunks < 1) chunks = 1;
    group_amax_kernel<<<dim3(chunks, static_cast<unsigned>(groups)), 256, 0, stream>>>(xv, n8, ws);
    rc = cuda_status(cudaGetLastError());
    if (rc) return rc;
    if (global) {
        global_amax_kernel<<<1, 256, 0, stream>>>(ws, groups);
        rc = cuda_status(cudaGetLastError());
        if (rc) return rc;
    }
    if (!transpose) {
        int cb = static_cast<int>((n8 + 255) / 256);
        const int cap = static_cast<int>((148 * 16 + groups - 1) / groups);
        if (cb > cap) cb = cap;
        if (cb < 1) cb = 1;
        group_convert_kernel<<<dim3(cb, static_cast<unsigned>(groups)), 256, 0, stream>>>(
            xv, n8, ws, reinterpret_cast<uint2 *>(xq), scale);
    } else {
        const int64_t ld = intfa_vt_ld(rows);
        const int64_t total = groups * ((ld + kPRows - 1) / kPRows);
        const unsigned grid = static_cast<unsigned>(total < 148 * 4 ? total : 148 * 4);
#define INTFA_TP(C8) group_convert_tp_kernel<C8><<<grid, kPThreads, 0, stream>>>(xv, rows, ld, groups, ws, xq, scale)
        switch (cols / 8) {
            case 1: INTFA_TP(1); break;
            case 2: INTFA_TP(2); break;
            case 4: INTFA_TP(4); break;
            case 8: INTFA_TP(8); break;
            case 16: INTFA_TP(16); break;
            case 32: INTFA_TP(32); break;
            default: {   // other multiples of 8 up to 256: the tile-per-block kernel
                const unsigned tiles = static_cast<unsigned>((ld + kTRows - 1) / kTRows);
                group_convert_t_kernel<<<dim3(tiles, static_cast<unsigned>(groups)), 256, 0, stream>>>(
                    xv, rows, cols, ld, ws, xq, scale);
            }
        }
#undef INTFA_TP
    }
    return cuda_status(cudaGetLastError());
}

}  // namespace intfa

// ------------------------------------------------------------------ C ABI ---

extern "C" int intfa_quantize_per_token(const void *x_f16, int64_t rows, int d, int8_t *x_q,
                                        float *scale, void *stream) {
    using namespace intfa;
    if (rows < 0) return INTFA_ERR_INVALID_ARG;
    if (rows > 0 && (!x_f16 || !x_q || !scale)) return INTFA_ERR_INVALID_ARG;
    if (!(d == 8 || d == 16 || d == 32 || d == 64 || d == 128 || d == 256)) return INTFA_ERR_UNSUPPORTED;
    if (rows > (INT64_MAX / 2) / d) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(x_f16) || (reinterpret_cast<uintptr_t>(x_q) & 7u) != 0 ||
        (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
        return INTFA_ERR_MISALIGNED;
    if (d >= 16 && !aligned16(x_q)) return INTFA_ERR_MISALIGNED;
    return launch_quantize_per_token(x_f16, rows, d, x_q, scale, static_cast<cudaStream_t>(stream));
}

extern "C" int intfa_quantize_per_token_bits(const void *x_f16, int64_t rows, int d, int bits, int8_t *x_q,
                                             float *scale, void *stream) {
    using namespace intfa;
    if (rows < 0 || bits < 2 || bits > 8) return INTFA_ERR_INVALID_ARG;
    if (rows > 0 && (!x_f16 || !x_q || !scale)) return INTFA_ERR_INVALID_ARG;
    if (!(d == 8 || d == 16 || d == 32 || d == 64 || d == 128 || d == 256)) return INTFA_ERR_UNSUPPORTED;
    if (rows > (INT64_MAX / 2) / d) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(x_f16) || (reinterpret_cast<uintptr_t>(x_q) & 7u) != 0 ||
        (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
        return INTFA_ERR_MISALIGNED;
    return launch_quantize_per_token_bits(x_f16, rows, d, bits, x_q, scale, static_cast<cudaStream_t>(stream));
}

extern "C" size_t intfa_quantize_per_tensor_workspace_size(int64_t groups) {
    if (groups <= 0) return 0;
    return intfa::round_up(static_cast<size_t>(groups) * sizeof(unsigned), 256);
}

extern "C" int64_t intfa_vt_ld(int64_t rows) { return rows <= 0 ? 0 : (rows + 15) / 16 * 16; }

extern "C" int intfa_quantize_per_tensor(const void *x_f16, int64_t groups, int64_t rows, int cols,
                                         int transpose, int8_t *x_q, float *scale,
                                         void *workspace, size_t workspace_bytes, void *stream) {
    using namespace intfa;
    if (groups < 0 || rows < 0 || cols <= 0) return INTFA_ERR_INVALID_ARG;
    if (transpose != 0 && transpose != 1) return INTFA_ERR_INVALID_ARG;
    if (cols % 8 != 0) return INTFA_ERR_UNSUPPORTED;
    if (transpose && cols > 256) return INTFA_ERR_UNSUPPORTED;
    if (groups == 0 || rows == 0) return INTFA_OK;
    if (groups > 65535) return INTFA_ERR_UNSUPPORTED;
    if (rows > (INT64_MAX / 4) / cols / groups) return INTFA_ERR_INVALID_ARG;
    if (!x_f16 || !x_q || !scale) return INTFA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < intfa_quantize_per_tensor_workspace_size(groups))
        return INTFA_ERR_WORKSPACE;
    if (!aligned16(x_f16) || !aligned16(x_q) || !aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
        return INTFA_ERR_MISALIGNED;
    return launch_quantize_per_tensor(x_f16, groups, rows, cols, transpose, x_q, scale, workspace,
                                      static_cast<cudaStream_t>(stream));
}

extern "C" int intfa_quantize_global(const void *x_f16, int64_t groups, int64_t rows, int cols, int transpose,
                                     int8_t *x_q, float *scale, void *workspace, size_t workspace_bytes,
                                     void *stream) {
    using namespace intfa;
    if (groups < 0 || rows < 0 || cols <= 0) return INTFA_ERR_INVALID_ARG;
    if (transpose != 0 && transpose != 1) return INTFA_ERR_INVALID_ARG;
    if (cols % 8 != 0) return INTFA_ERR_UNSUPPORTED;
    if (transpose && cols > 256) return INTFA_ERR_UNSUPPORTED;
    if (groups == 0 || rows == 0) return INTFA_OK;
    if (groups > 65535) return INTFA_ERR_UNSUPPORTED;
    if (rows > (INT64_MAX / 4) / cols / groups) return INTFA_ERR_INVALID_ARG;
    if (!x_f16 || !x_q || !scale) return INTFA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < intfa_quantize_per_tensor_workspace_size(groups))
        return INTFA_ERR_WORKSPACE;
    if (!aligned16(x_f16) || !aligned16(x_q) || !aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
        return INTFA_ERR_MISALIGNED;
    return launch_quantize_per_tensor(x_f16, groups, rows, cols, transpose, x_q, scale, workspace,
                                      static_cast<cudaStream_t>(stream), true);
}

// ------------------------------------------- per tensor, no allocation ---
//
// For callers that cannot allocate device memory themselves (see
// intfa_quantize_per_tensor_noalloc in include/intfa.h): the per-group abs-max
// scratch of the per-tensor quantiser lives in this file-scope device array
// instead of a caller workspace.  Every GPU that loads the library holds it
// until the process exits.  Host code must not pass the symbol itself to a
// kernel (on the host it only names a stand-in); its device address is looked
// up once per device with cudaGetSymbolAddress and cached.

static __device__ __align__(256) unsigned g_noalloc_amax[INTFA_NOALLOC_MAX_GROUPS];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_amax on the current device (set-up on first use).
int noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return intfa::cuda_status(cudaErrorInvalidDevice);
    if (dev < 0 || dev >= kMaxDevices) return INTFA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_amax);
        if (e != cudaSuccess || p == nullptr) return intfa::cuda_status(e == cudaSuccess ? cudaErrorUnknown : e);
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return INTFA_OK;
}

}  // namespace

extern "C" int intfa_quantize_per_tensor_noalloc(const void *x_f16, int64_t groups, int64_t rows,
                                                 int cols, int transpose, int8_t *x_q, float *scale,
                                                 void *stream) {
    using namespace intfa;
    if (groups < 0 || rows < 0 || cols <= 0) return INTFA_ERR_INVALID_ARG;
    if (transpose != 0 && transpose != 1) return INTFA_ERR_INVALID_ARG;
    if (cols % 8 != 0) return INTFA_ERR_UNSUPPORTED;
    if (transpose && cols > 256) return INTFA_ERR_UNSUPPORTED;
    if (groups > INTFA_NOALLOC_MAX_GROUPS) return INTFA_ERR_UNSUPPORTED;   // beyond the built-in scratch
    if (groups == 0 || rows == 0) return INTFA_OK;
    if (rows > (INT64_MAX / 4) / cols / groups) return INTFA_ERR_INVALID_ARG;
    if (!x_f16 || !x_q || !scale) return INTFA_ERR_INVALID_ARG;
    if (!aligned16(x_f16) || !aligned16(x_q) || (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
        return INTFA_ERR_MISALIGNED;
    void *scratch = nullptr;
    const int rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    // The launcher clears the scratch (cudaMemsetAsync) before the abs-max pass.
    return launch_quantize_per_tensor(x_f16, groups, rows, cols, transpose, x_q, scale, scratch,
                                      static_cast<cudaStream_t>(stream));
}
