/*
 * intfa.h -- C ABI of libintfa: INT8-quantised attention forward pass on
 * NVIDIA B200 (sm_100a), in the style of INT-FlashAttention.
 *
 * The method (sources are web pages; each entry point cites its passage):
 *   - INT-FlashAttention: Enabling Flash Attention for INT8 Quantization,
 *     abstract: an INT8 FlashAttention forward pass with token-level
 *     (per-row) quantisation of Q and K.
 *   - IntAttention: A Fully Integer Attention Pipeline for Efficient Edge
 *     Inference, section 2.1: the symmetric quantiser (eq. 3), integer
 *     logits with a float rescale (eq. 4), O ~= s_V P V_hat (eq. 5);
 *     section 2.2: the row-max-stable softmax (eq. 6); section 3.2:
 *     probabilities multiplied by 127 and stored as signed INT8.
 *   - FlashAttention-3 (arXiv 2407.08608), abstract: block-wise softmax
 *     interleaved with the two matmuls (running max and running sum).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, unless the
 *     name ends in _host.  The library allocates no device memory; scratch
 *     space is a caller-provided workspace whose size a *_workspace_size
 *     function returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Calls are asynchronous on that stream; INTFA_OK means the
 *     arguments were valid and the kernels were launched.  Faults inside a
 *     kernel surface at the caller's next synchronisation.
 *   - Arguments are checked on the host before anything is launched; a
 *     failed check returns an error code and launches nothing.
 *   - Inputs must be finite; NaN or Inf inputs give unspecified results.
 *   - Every entry point is thread-safe and keeps no state between calls,
 *     except the device-side status word read by intfa_device_status.
 */
#ifndef INTFA_H_
#define INTFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
typedef enum {
    INTFA_OK = 0,
    INTFA_ERR_INVALID_ARG = 1,    /* null pointer, negative or zero size, overflow */
    INTFA_ERR_UNSUPPORTED = 2,    /* a shape the kernels do not implement (e.g. d) */
    INTFA_ERR_MISALIGNED = 3,     /* a pointer is not 16-byte aligned */
    INTFA_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed */
    INTFA_ERR_DEVICE_TIMEOUT = 5, /* a kernel gave up on a bounded wait (see
                                     intfa_device_status) */
    INTFA_ERR_WORKSPACE = 6       /* workspace missing or too small */
} intfa_status;

/* Static description of a status code; never NULL. */
const char *intfa_status_string(int status);

/*
 * Per-token symmetric INT8 quantisation (IntAttention section 2.1, eq. 3,
 * applied to each token row as INT-FlashAttention's abstract specifies).
 *
 *   x_f16  : fp16 [rows][d], row-major, 16-byte aligned.
 *   x_q    : int8 [rows][d] out, 16-byte aligned (8-byte for d == 8).
 *   scale  : fp32 [rows] out.
 * For each row: s = max_k |x_k| / 127 (one IEEE fp32 division),
 * x_q[k] = clamp(round-half-even(x_k / s), -127, 127) with x_k / s the IEEE
 * fp32 quotient; an all-zero row gives s = 0 and codes 0.  Bit-exact.
 * d must be one of 8, 16, 32, 64, 128, 256; rows >= 0 (0 is a no-op).
 */
int intfa_quantize_per_token(const void *x_f16, int64_t rows, int d, int8_t *x_q,
                             float *scale, void *stream);

/*
 * Per-tensor symmetric INT8 quantisation (IntAttention section 2.1, eq. 3,
 * one scale per L x d tensor, as that section applies it to V).
 *
 *   x_f16  : fp16 [groups][rows][cols], row-major, 16-byte aligned.
 *   scale  : fp32 [groups] out: s_g = max |x| over group g / 127.
 *   x_q    : int8 out, codes as in intfa_quantize_per_token with s_g.
 *            transpose == 0: [groups][rows][cols] (same layout as x).
 *            transpose == 1: [groups][cols][ld] with ld = intfa_vt_ld(rows):
 *            the transpose of each group, rows padded with zero codes up to
 *            ld.  This is the V_hat^T layout intfa_attention_fwd reads.
 *   workspace : device scratch of at least
 *            intfa_quantize_per_tensor_workspace_size(groups) bytes, 16-byte
 *            aligned; its contents on entry do not matter.
 * cols must be a multiple of 8 and, with transpose, at most 256.
 */
/*
 * Per-token quantisation with b-bit symmetric codes (the pages' remark that
 * the token-level scheme extends to INT4; IntAttention eq. 3 with 127
 * replaced by qmax = 2^(b-1) - 1): s = fl32(max|x| / qmax), codes
 * clamp(RNE(x / s), -qmax, qmax) stored one per int8, so the INT8 attention
 * entry points take them unchanged (tcgen05 has no narrower integer MMA).
 * bits in 2..8 (8 gives intfa_quantize_per_token's codes and scales);
 * other arguments and errors as intfa_quantize_per_token.
 */
int intfa_quantize_per_token_bits(const void *x_f16, int64_t rows, int d, int bits, int8_t *x_q,
                                  float *scale, void *stream);

size_t intfa_quantize_per_tensor_workspace_size(int64_t groups);
int64_t intfa_vt_ld(int64_t rows);
int intfa_quantize_per_tensor(const void *x_f16, int64_t groups, int64_t rows, int cols,
                              int transpose, int8_t *x_q, float *scale, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * One scale for the whole tensor (IntAttention section 2.1, eq. 3 applied to
 * all groups together: "per-tensor" read as one scale for the whole V
 * tensor rather than one per L x d head): s = fl32(max over all groups of
 * max|x| / 127), the
 * codes of every group with that s, in the same per-group layout as
 * intfa_quantize_per_tensor (transpose 0 or 1), and s written to each of the
 * `groups` scale slots, so that the attention entry points (one s_V per head)
 * take it unchanged.  Arguments, workspace and errors as
 * intfa_quantize_per_tensor.
 */
int intfa_quantize_global(const void *x_f16, int64_t groups, int64_t rows, int cols, int transpose,
                          int8_t *x_q, float *scale, void *workspace, size_t workspace_bytes,
                          void *stream);

/*
 * Per-tensor quantisation without any device allocation.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory themselves and therefore cannot supply the workspace that
 * intfa_quantize_per_tensor needs -- for instance a plug-in running inside a
 * host application whose memory pool owns all device memory, or a
 * latency-critical caller that must not take the device-wide synchronisation
 * of cudaMalloc / cudaFree.
 *
 * Same arguments, results and layout rules as intfa_quantize_per_tensor
 * (bit-identical output), minus the workspace.  The per-group scratch is a
 * fixed array of INTFA_NOALLOC_MAX_GROUPS 32-bit words (16 KiB) compiled into
 * the library; every GPU that loads the library holds it until the process
 * exits.  groups > INTFA_NOALLOC_MAX_GROUPS returns INTFA_ERR_UNSUPPORTED
 * before touching the device.  The first call on each device looks up the
 * array's device address (a one-time set-up, which may load the module); make
 * that first call before any stream capture.  All calls share the one array:
 * the call clears what it needs before use, but calls that overlap on the GPU
 * (on different streams, or from several threads without ordering) race on it
 * and give wrong results -- serialise them.  Nothing here calls cudaMalloc,
 * cudaFree or any allocating routine.  The looked-up address is kept for the
 * life of the process: after cudaDeviceReset on a device the library must not
 * be used on that device again in the same process (the module may load at
 * another address; the same holds for intfa_forward_host's copy streams).
 */
#define INTFA_NOALLOC_MAX_GROUPS 4096
int intfa_quantize_per_tensor_noalloc(const void *x_f16, int64_t groups, int64_t rows, int cols,
                                      int transpose, int8_t *x_q, float *scale, void *stream);

/*
 * Fused INT8 attention forward pass (INT-FlashAttention abstract; IntAttention
 * eqs. 4-6, section 3.2 and eq. 5; FlashAttention-3's block-wise online
 * softmax), one kernel:
 *   S = Q_hat K_hat^T (INT8 x INT8 -> INT32, tcgen05 tensor cores, TMEM)
 *   t_ij = S_ij s_Q[i] s_K[j] / sqrt(d), keys masked j > i when causal
 *   per key block of 128: running max m, p = exp(t - m), P_hat = RNE(127 p),
 *   O_blk = P_hat V_hat (INT8 x INT8 -> INT32), acc = alpha acc + O_blk,
 *   l = alpha l + sum p, alpha = exp(m_old - m_new)
 *   O = s_V acc / (127 l), written as fp16.
 *
 *   Q_q, K_q : int8 [B][H][L][d] (from intfa_quantize_per_token), 16-B aligned.
 *   Vt_q     : int8 [B][H][d][intfa_vt_ld(L)] = V_hat transposed per head
 *              (from intfa_quantize_per_tensor with transpose = 1), 16-B aligned.
 *   s_Q, s_K : fp32 [B][H][L]; s_V : fp32 [B][H] (one scale per head).
 *   O_f16    : fp16 [B][H][L][d] out, 16-byte aligned.
 *   d in {64, 128}; L >= 1 (any value; the last key/query block is masked);
 *   causal in {0, 1} (square, top-left aligned: key j visible to query i iff
 *   j <= i).  Returns INTFA_ERR_DEVICE_TIMEOUT only via intfa_device_status.
 */
int intfa_attention_fwd(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                        const float *s_Q, const float *s_K, const float *s_V, int B, int H,
                        int L, int d, int causal, void *O_f16, void *stream);

/*
 * The same fused attention with V_hat in its natural layout: V_q int8
 * [B][H][L][d] (intfa_quantize_per_tensor with groups = B*H and
 * transpose = 0), 16-byte aligned; every other argument as in
 * intfa_attention_fwd, and the output is bit-identical to it on the same
 * codes.  The kernel's P V product reads the V_hat tile N-major, so no
 * transposed copy of V_hat is made; intfa_forward takes this path.
 */
int intfa_attention_fwd_vrows(const int8_t *Q_q, const int8_t *K_q, const int8_t *V_q,
                              const float *s_Q, const float *s_K, const float *s_V, int B, int H,
                              int L, int d, int causal, void *O_f16, void *stream);

/*
 * The same fused attention with Q given in fp16: each 128-query tile is
 * quantised per token inside the kernel (IntAttention section 2.1, eq. 3,
 * token-level as INT-FlashAttention's abstract specifies; bit-identical codes
 * and scales to intfa_quantize_per_token), so Q_hat never travels through
 * HBM.  The pages describe quantisation and attention as separate steps; this
 * fusion is an implementation choice of this library.
 *
 *   Q_f16   : fp16 [B][H][L][d], 16-byte aligned.
 *   s_Q_out : fp32 [B][H][L] out (the per-token scales), or NULL.
 *   Other arguments, results and error behaviour as intfa_attention_fwd; O
 *   equals intfa_attention_fwd's output on intfa_quantize_per_token(Q) bit
 *   for bit.
 */
int intfa_attention_fwd_q16(const void *Q_f16, const int8_t *K_q, const int8_t *Vt_q,
                            const float *s_K, const float *s_V, int B, int H, int L, int d,
                            int causal, void *O_f16, float *s_Q_out, void *stream);

/*
 * The fused attention of intfa_attention_fwd with the other reading of the
 * row sum: l = alpha l + sum_j P_hat_ij / 127 (the sum of the INT8 P codes,
 * IntAttention section 3.2 quantising P before the value product) instead of
 * the sum of the unquantised p.  O = s_V acc / (127 l) is then the P-code
 * weighted mean of V_hat.  Arguments, layouts and errors as
 * intfa_attention_fwd.
 */
int intfa_attention_fwd_codesum(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                                const float *s_Q, const float *s_K, const float *s_V, int B, int H,
                                int L, int d, int causal, void *O_f16, void *stream);

/*
 * The fused attention of intfa_attention_fwd with the P-code range and the
 * row-sum reading chosen by the caller.
 *
 *   p_levels   : 127 -- P_hat = RNE(127 p) stored as INT8 (IntAttention
 *                section 3.2, the INT-FlashAttention pipeline; the codes of
 *                intfa_attention_fwd);
 *                255 -- P_hat = RNE(255 p) stored as UINT8 and multiplied as
 *                unsigned tensor-core operands (the unsigned scheme of
 *                IntAttention's Table 5 ablation, which spends all 256 codes
 *                on p in [0, 1]).  O = s_V (P_hat V_hat) / (p_levels l).
 *   lsum_codes : 0 -- l from the unquantised p (as intfa_attention_fwd);
 *                1 -- l from the codes, sum P_hat / p_levels (as
 *                intfa_attention_fwd_codesum when p_levels = 127).
 *   Other arguments, layouts and error behaviour as intfa_attention_fwd;
 *   INTFA_ERR_INVALID_ARG for any other p_levels or lsum_codes.
 *   (127, 0) and (127, 1) give output bit-identical to intfa_attention_fwd
 *   and intfa_attention_fwd_codesum.
 */
int intfa_attention_fwd_pcodes(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                               const float *s_Q, const float *s_K, const float *s_V, int B, int H,
                               int L, int d, int causal, int p_levels, int lsum_codes, void *O_f16,
                               void *stream);

/*
 * The fused attention of intfa_attention_fwd with group-wise Q and K scales
 * (IntAttention section 3.3: per-block quantisation; the scales of each
 * group factor out of Q_hat K_hat^T exactly as per-token scales do): one scale
 * per block of scale_block consecutive tokens of a head.
 *
 *   s_Q, s_K    : fp32 [B][H][ceil(L / scale_block)]; the scale of token i is
 *                 s[i / scale_block].  Codes as from intfa_quantize_per_tensor
 *                 with groups = B*H*L/scale_block (L a multiple of scale_block).
 *   scale_block : a power of two, 1 .. 65536 (1 = intfa_attention_fwd).
 *   Other arguments, layouts and error behaviour as intfa_attention_fwd;
 *   INTFA_ERR_INVALID_ARG for any other scale_block.
 */
int intfa_attention_fwd_blockscale(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                                   const float *s_Q, const float *s_K, const float *s_V, int B,
                                   int H, int L, int d, int causal, int scale_block, void *O_f16,
                                   void *stream);

/*
 * IndexSoftmax attention (IntAttention: A Fully Integer Attention Pipeline for
 * Efficient Edge Inference, section 3.1 eqs. 7-10, section 3.2, and eq. 5 for
 * the value path) with per-tensor scales, section 3.3's default
 * configuration.  Per head (scales s_Q, s_K, s_V):
 *   A_hat  = Q_hat K_hat^T (INT8 x INT8 -> INT32); m_i = row max over visible keys
 *   c_int  = rint((c sqrt(d)) / (s_Q s_K)) in fp64, at least 1   (eq. 8)
 *   idx_ij = floor(min(m_i - A_hat_ij, c_int) (2^b - 1) / c_int)  (eqs. 9-10)
 *   E_ij   = LUT[idx_ij], LUT[k] = rint(255 exp(-c k / (2^b - 1))) (UINT8 P x 255)
 *   O_i    = s_V (sum_j E_ij V_hat_j) / (sum_j E_ij), written as fp16
 * The row max covers the whole row before any lookup (two passes over the
 * keys); the integer sums are exact.  The pages normalise the 8-bit
 * probabilities before P V; here the same quotient is taken after it, which
 * avoids rounding normalised probabilities below 1/255 to zero on long rows.
 *
 *   Q_q, K_q : int8 [B][H][L][d], per-tensor codes (intfa_quantize_per_tensor
 *              with groups = B*H, transpose = 0), 16-B aligned.
 *   Vt_q     : int8 [B][H][d][intfa_vt_ld(L)] as for intfa_attention_fwd.
 *   s_Q, s_K, s_V : fp32 [B][H] (one scale per head each).
 *   c, b     : clip threshold (0 < c < 1e30) and table bits (1 .. 8); the
 *              pages recommend (b, c) = (5, 6.6).
 *   O_f16    : fp16 [B][H][L][d] out, 16-byte aligned.
 *   m_out, l_out : int32 [B][H][L] out or NULL: the integer row max of A_hat
 *              and the integer row sum of E (exact, for checking).
 *   d in {64, 128}; 1 <= L <= 65536 (int32 accumulation: 255 * 127 * L <
 *   2^31); causal in {0, 1}.  INTFA_ERR_INVALID_ARG / UNSUPPORTED /
 *   MISALIGNED for bad arguments, INTFA_ERR_CUDA for a failed launch; a
 *   device-side timeout shows in intfa_device_status.
 */
int intfa_index_attention_fwd(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                              const float *s_Q, const float *s_K, const float *s_V, int B,
                              int H, int L, int d, int causal, double c, int b, void *O_f16,
                              int32_t *m_out, int32_t *l_out, void *stream);

/*
 * Decode: one query per head against an INT8 key / value cache, the online
 * form of intfa_attention_fwd (INT-FlashAttention abstract; IntAttention eqs.
 * 3-6, section 3.2, eq. 5) for a single query row, with the keys cut into
 * `splits` ranges of split_len = ceil(ceil(L / 128) / splits) * 128 keys that
 * each run the block-wise steps on their own (running max, P codes against
 * that range's running max) and are merged at the end:
 *   M = max_s m_s,  O = s_V sum_s e^(m_s - M) acc_s / (127 sum_s e^(m_s - M) l_s).
 * The query is quantised per token inside the kernel (bit-identical to
 * intfa_quantize_per_token).  No mask: every cache entry is visible.
 *
 *   q_f16  : fp16 [B][H][d], 16-byte aligned.
 *   K_q    : int8 [B][H][L][d] per-token codes (intfa_quantize_per_token),
 *            s_K fp32 [B][H][L].
 *   V_q    : int8 [B][H][L][d] per-head codes, row-major
 *            (intfa_quantize_per_tensor, groups = B*H, transpose = 0), s_V
 *            fp32 [B][H].
 *   splits : 1 .. 65535 ranges per head (ranges past the end are empty).
 *   O_f16  : fp16 [B][H][d] out.
 *   workspace : device scratch of intfa_decode_workspace_size(B, H, d,
 *            splits) bytes, 16-byte aligned (the per-range partial results).
 *   d in {64, 128}; 1 <= L <= 2^24; B*H <= 65535.
 */
size_t intfa_decode_workspace_size(int B, int H, int d, int splits);
int intfa_decode_fwd(const void *q_f16, const int8_t *K_q, const float *s_K, const int8_t *V_q,
                     const float *s_V, int B, int H, int L, int d, int splits, void *O_f16,
                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * Debug: the integer logits S = Q_hat K_hat^T (IntAttention eq. 4) for every
 * head, int32 [B][H][L][L], computed by the same TMA + tcgen05 path the fused
 * kernel uses for its first contraction.  Same layout rules as
 * intfa_attention_fwd for Q_q and K_q; S must be 16-byte aligned.
 */
int intfa_debug_qk(const int8_t *Q_q, const int8_t *K_q, int B, int H, int L, int d,
                   int32_t *S, void *stream);

/*
 * Debug: intfa_attention_fwd (same kernel, same arithmetic, same O) that also
 * writes the integer logits S = Q_hat K_hat^T (IntAttention eq. 4) as the
 * kernel's softmax recovers them from its tensor-memory accumulator, int32
 * [B][H][L][L].  Entries of key blocks the kernel never computes (past the
 * diagonal block under causal masking) are left untouched.  Arguments as
 * intfa_attention_fwd plus S (16-byte aligned); B*H*L*L must not exceed
 * 2^28 (INTFA_ERR_UNSUPPORTED otherwise).
 */
int intfa_debug_attention_scores(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                                 const float *s_Q, const float *s_K, const float *s_V, int B,
                                 int H, int L, int d, int causal, void *O_f16, int32_t *S,
                                 void *stream);

/*
 * Test of the bounded waits (no counterpart in the pages): launches the
 * fused attention kernel (d = 64) in a form that issues no copy and no
 * tensor-core operation, with every wait capped at cap_cycles clock cycles,
 * so that each role's first wait runs out.  The kernel records the wait site
 * in the device status word, frees its tensor memory and returns; afterwards
 * intfa_device_status reports INTFA_ERR_DEVICE_TIMEOUT and the site, and the
 * device stays usable.  Arguments as intfa_attention_fwd (the buffers must
 * be valid: their tensor maps are built but never read) with d = 64;
 * cap_cycles in [1000, 2^32]; O_f16 is left untouched.
 */
int intfa_debug_wait_timeout(const int8_t *Q_q, const int8_t *K_q, const int8_t *Vt_q,
                             const float *s_Q, const float *s_K, const float *s_V, int B, int H,
                             int L, int d, int causal, void *O_f16, int64_t cap_cycles,
                             void *stream);

/*
 * Whole hot path on device buffers: quantise Q and K per token, V per head
 * (codes kept in V's [B][H][L][d] layout), then the fused attention
 * (intfa_attention_fwd_vrows).  V's quantiser runs on a stream of the
 * library's own (one per device, made with two events on the first call, like
 * intfa_forward_host's copy streams) beside Q's and K's on `stream`, which
 * waits for it before the attention; make the first call on a device before
 * any stream capture.  Calls are serialised by a host mutex while they queue
 * their work.  Q, K, V, O: fp16 [B][H][L][d]
 * device pointers; workspace: intfa_forward_workspace_size(B, H, L, d) bytes of
 * device memory, 256-byte aligned.  Optional outputs of the quantisation live
 * in the workspace at the offsets intfa_forward_workspace_layout reports.
 */
size_t intfa_forward_workspace_size(int B, int H, int L, int d);
/* offsets[0..5] = byte offsets of Q_q, K_q, V_q ([B][H][L][d], untransposed),
 * s_Q, s_K, s_V inside the workspace; returns INTFA_OK or
 * INTFA_ERR_INVALID_ARG. */
int intfa_forward_workspace_layout(int B, int H, int L, int d, size_t offsets[6]);
int intfa_forward(const void *Q_f16, const void *K_f16, const void *V_f16, int B, int H, int L,
                  int d, int causal, void *O_f16, void *workspace, size_t workspace_bytes,
                  void *stream);

/*
 * The same from HOST memory: copies Q, K, V (fp16, host, pinned for
 * asynchronous copies) to the device, runs the path of intfa_forward and
 * copies O back to O_f16_host.  workspace:
 * intfa_forward_host_workspace_size(B, H, L, d) bytes of device memory,
 * 256-byte aligned.  Asynchronous on `stream`: O_f16_host is valid after the
 * stream is synchronised.  The heads are processed in chunks (each half of
 * the heads left, at least 4 MiB of fp16 per tensor): chunk c's input copies, its
 * quantisation + attention and its output copy overlap with the other chunks'
 * copies in the opposite direction.  The copies run on two streams of the
 * library's own (one pair per device, created on the first call and kept for
 * the life of the process); calls are serialised by a host mutex while they
 * queue their work.  Output bit-identical to intfa_forward.
 */
size_t intfa_forward_host_workspace_size(int B, int H, int L, int d);
int intfa_forward_host(const void *Q_f16_host, const void *K_f16_host, const void *V_f16_host,
                       int B, int H, int L, int d, int causal, void *O_f16_host,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * Device-side status: every wait inside the fused kernel is bounded; a kernel
 * that gives up records a nonzero word and returns without hanging the GPU.
 * Synchronises the current device, returns INTFA_OK if the word is zero,
 * INTFA_ERR_DEVICE_TIMEOUT otherwise (and the word in *word if non-NULL);
 * clear != 0 resets it to zero.
 */
int intfa_device_status(int clear, uint32_t *word);

#ifdef __cplusplus
}
#endif

#endif /* INTFA_H_ */
