// quantize.cu -- symmetric INT8 quantisation kernels (IntAttention: A Fully
// Integer Attention Pipeline for Efficient Edge Inference, section 2.1,
// eq. 3: s = max|x| / 127, x ~= s x_hat, zero-point 0), per token row for Q
// and K (INT-FlashAttention, abstract: token-level quantisation) and per
// L x d tensor for V.
//
// Both are HBM-bound streaming kernels: 16-byte vector loads of 8 fp16
// values per thread, warp-shuffle row reductions, 8-byte code stores.
//
// Rounding contract (bit-exact with the definition): s = fl32(amax / 127)
// by an IEEE division; the code is RNE(fl32(x / s)) clamped to +-127.  The
// per-element quotient is formed as y = x * r with r = rcp.approx(s)
// (relative error <= 2^-23): |y - x/s| <= 127 (2^-23 + 2^-24) <= 2.3e-5 and
// |fl32(x/s) - x/s| <= 7.6e-6, so y and fl32(x/s) round to the same integer
// unless x/s lies within ~3.1e-5 of a half-integer; when y is within 1e-3 of
// one, the IEEE quotient __fdiv_rn(x, s) is used instead.  The result is
// therefore identical to rounding the IEEE quotient, at one multiply per
// element.
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
    uint2 *qv = reinterpret_cast<uint2 *>(xq);
    const int rows_per_block = 256 / (d / 8);
    const int grid = grid_for(rows, rows_per_block);
    switch (d) {
        case 8: quant_per_token_kernel<1><<<grid, 256, 0, stream>>>(xv, rows, qv, scale); break;
        case 16: quant_per_token_kernel<2><<<grid, 256, 0, stream>>>(xv, rows, qv, scale); break;
        case 32: quant_per_token_kernel<4><<<grid, 256, 0, stream>>>(xv, rows, qv, scale); break;
        case 64: quant_per_token_kernel<8><<<grid, 256, 0, stream>>>(xv, rows, qv, scale); break;
        case 128: quant_per_token_kernel<16><<<grid, 256, 0, stream>>>(xv, rows, qv, scale); break;
        case 256: quant_per_token_kernel<32><<<grid, 256, 0, stream>>>(xv, rows, qv, scale); break;
        default: return INTFA_ERR_UNSUPPORTED;
    }
    return cuda_status(cudaGetLastError());
}

int launch_quantize_per_tensor(const void *x, int64_t groups, int64_t rows, int cols,
                               int transpose, int8_t *xq, float *scale, void *workspace,
                               cudaStream_t stream, bool global) {
    if (groups == 0) return INTFA_OK;
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
        const unsigned tiles = static_cast<unsigned>((ld + kTRows - 1) / kTRows);
        group_convert_t_kernel<<<dim3(tiles, static_cast<unsigned>(groups)), 256, 0, stream>>>(
            xv, rows, cols, ld, ws, xq, scale);
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
