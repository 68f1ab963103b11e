// internal.h -- host-side helpers shared by the libintfa translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/intfa.h"

namespace intfa {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return INTFA_OK;
    (void)cudaGetLastError();  // clear the sticky-free error so later calls are not poisoned
    return INTFA_ERR_CUDA;
}

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launchers implemented in quantize.cu / attention.cu (arguments already checked).
int launch_quantize_per_token(const void *x, int64_t rows, int d, int8_t *xq, float *scale,
                              cudaStream_t stream);
// global: one scale over all groups (written to every group's slot).
int launch_quantize_per_tensor(const void *x, int64_t groups, int64_t rows, int cols,
                               int transpose, int8_t *xq, float *scale, void *workspace,
                               cudaStream_t stream, bool global = false);
// sshift: one scale per 2^sshift consecutive tokens of Q and K (0: per token).
int launch_attention_fwd(const int8_t *Qq, const int8_t *Kq, const int8_t *Vt,
                         const float *sQ, const float *sK, const float *sV, int B, int H, int L,
                         int d, int causal, void *O, cudaStream_t stream, int sshift = 0);
// Same, with V_hat in its natural layout Vq [B][H][L][d] (no transpose).
int launch_attention_fwd_vrows(const int8_t *Qq, const int8_t *Kq, const int8_t *Vq, const float *sQ,
                               const float *sK, const float *sV, int B, int H, int L, int d, int causal,
                               void *O, cudaStream_t stream);
int launch_attention_fwd_q16(const void *Qh, const int8_t *Kq, const int8_t *Vt, const float *sK,
                             const float *sV, int B, int H, int L, int d, int causal, void *O,
                             float *sQ_out, cudaStream_t stream);
// Test instantiations of the fused attention kernel: mode 1 also writes the
// recovered S of every block to dbg [B*H][L][L] (int32); mode 2 (d = 64 only)
// issues no load and no MMA, so that every bounded wait runs out after `cap`
// clock cycles.
int launch_attention_debug(int mode, const int8_t *Qq, const int8_t *Kq, const int8_t *Vt, const float *sQ,
                           const float *sK, const float *sV, int B, int H, int L, int d, int causal, void *O,
                           cudaStream_t stream, long long cap, int32_t *dbg);
// The IndexSoftmax kernel's status word (index_attention.cu); clear resets it.
int read_index_status(int clear, uint32_t *word);
// The decode kernels' status word (decode.cu); clear resets it.
int read_decode_status(int clear, uint32_t *word);

}  // namespace intfa
