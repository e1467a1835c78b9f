/*
 * sa3.h -- C ABI of libsa3: microscaled-FP4 attention forward on B200
 * (sm_100a).
 *
 * The method ("SageAttention3: Microscaling FP4 Attention for Inference and
 * An Exploration of 8-Bit Training", abstract) computes attention on the
 * Blackwell FP4 tensor cores: K is first smoothed by subtracting its mean
 * over tokens, which leaves softmax attention unchanged ("SageAttention:
 * Accurate 8-Bit Attention for Plug-and-play Inference Acceleration",
 * section "Approach"); Q, K and V are quantized to FP4 E2M1 with one E4M3
 * scale per 16 elements; S = Q K^T and O = P V run as block-scaled FP4
 * matrix products, with P quantized the same way once per 128-token KV
 * block against the running row maximum of a blockwise online softmax.
 *
 * Conventions for every call:
 *   - every pointer argument is a DEVICE pointer (cudaMalloc'ed or from a
 *     caching allocator) unless stated otherwise; the library never
 *     allocates, frees or keeps a reference to caller memory;
 *   - calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream); a return of SA3_OK means the arguments were valid
 *     and the kernels were enqueued, not that they have finished;
 *   - shapes: B, H >= 1; N >= 1; d in {64, 128}; B*H*N_p*d/2 < 2^31
 *     where N_p = N rounded up to a multiple of 128;
 *   - Q, K, V and the output are bf16, contiguous [B][H][N][d], 16-byte
 *     aligned;
 *   - quantizer outputs need 16-byte alignment.  When all the code outputs
 *     (q/k codes, V^T codes or FP16 V^T) are 32-byte aligned, as any
 *     cudaMalloc or torch allocation is, the quantizer writes 32-byte pieces
 *     in one store each, which is faster for the 8-bit variant.  The bytes
 *     written are the same either way;
 *   - the library is thread-safe for concurrent calls on different streams
 *     as long as their workspaces differ;
 *   - the first call of each kernel on a device sets that kernel's
 *     attributes, once.  Make it outside stream capture.  After it, the
 *     calls only enqueue kernels, with no allocation, synchronization or
 *     attribute call, so they can be recorded into a CUDA graph (stream
 *     capture) and replayed with new inputs in the same buffers;
 *   - no call's outputs may share bytes with its inputs (or its
 *     workspace): some CTAs still read inputs while others write, and the
 *     quantizer's second kernel starts loading K while the first may still
 *     be writing.  Such a call is rejected, including an in-place
 *     attention call whose output aliases the Q it quantizes on load.
 *
 * Error behaviour: arguments are checked before any launch; a bad argument
 * returns SA3_ERR_INVALID_ARG (null pointer, misalignment, non-positive
 * size, workspace too small, an output overlapping an input) or
 * SA3_ERR_UNSUPPORTED (d not 64/128, size limits) and enqueues nothing.
 * A failed launch returns SA3_ERR_CUDA.
 * Device-side waits are bounded; if one gives up, the kernel records
 * SA3_ERR_TIMEOUT in a device status word, releases what it holds and
 * returns; sa3_device_status() reports it.
 */
#ifndef SA3_H
#define SA3_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t */

typedef enum {
    SA3_OK = 0,
    SA3_ERR_INVALID_ARG = 1,
    SA3_ERR_UNSUPPORTED = 2,
    SA3_ERR_CUDA = 3,
    SA3_ERR_TIMEOUT = 4
} sa3_status;

/*
 * Quantized operands produced by sa3_quantize_qkv and consumed by
 * sa3_attn_fwd.  All device pointers, caller-owned, sizes from the helpers
 * below.  Layouts (bh = b*H + h, N_p = sa3_padded_len(N)):
 *
 *   q_fp4, k_fp4  u8 [B*H][N_p][d/2]: E2M1 codes, row-major, element 2i in
 *                 the low nibble of byte i, element 2i+1 in the high one.
 *   vt_fp4        u8 [B*H][d][N_p/2]: V transposed (channel-major), same
 *                 packing along tokens.
 *   q_sf, k_sf    E4M3 scale of the 16 elements (t, 16c .. 16c+15) stored at
 *                   (((bh*(N_p/128) + t/128)*(d/64) + c/4) * 512
 *                    + 16*(t%32) + 4*((t%128)/32) + c%4
 *                 i.e. 512-byte atoms of 128 tokens x 4 scales in the order
 *                 the tensor core's block-scaled MMA reads them.
 *   vt_sf         E4M3 scale of the 16 tokens (16u .. 16u+15) of channel c:
 *                   (bh*(N_p/64) + u/4) * 512 + 16*(c%32) + 4*(c/32) + u%4
 *                 (channels padded to 128; padding channels hold 0).
 *   k_mean        fp32 [B*H][d]: the mean of K over its N tokens.
 *
 * Tokens t >= N have code 0 and scale 0.  A block whose scale rounds to 0
 * has all codes 0.
 */
typedef struct sa3_qkv_fp4 {
    void *q_fp4;
    void *q_sf;
    void *k_fp4;
    void *k_sf;
    void *vt_fp4;
    void *vt_sf;
    float *k_mean;
} sa3_qkv_fp4;

/* ---- sizes (bytes); header-only helpers, not exported ---------------- */
static inline int64_t sa3_padded_len(int64_t N) { return (N + 127) / 128 * 128; }
static inline int64_t sa3_qk_fp4_bytes(int64_t B, int64_t H, int64_t N, int64_t d)
{ return B * H * sa3_padded_len(N) * d / 2; }
static inline int64_t sa3_qk_sf_bytes(int64_t B, int64_t H, int64_t N, int64_t d)
{ return B * H * sa3_padded_len(N) * d / 16; }
static inline int64_t sa3_vt_fp4_bytes(int64_t B, int64_t H, int64_t N, int64_t d)
{ return B * H * d * sa3_padded_len(N) / 2; }
static inline int64_t sa3_vt_sf_bytes(int64_t B, int64_t H, int64_t N, int64_t d)
{ (void)d; return B * H * sa3_padded_len(N) * 8; }
static inline int64_t sa3_kmean_bytes(int64_t B, int64_t H, int64_t d) { return B * H * d * 4; }
/* Scratch for the K-mean reduction: fp64 partial sums over chunks of
 * sa3_kmean_chunk(N) tokens (a multiple of 512 chosen so that there are at
 * most 16 chunks). */
static inline int64_t sa3_kmean_chunk(int64_t N) { return 512 * (((N + 511) / 512 + 15) / 16); }
static inline int64_t sa3_kmean_nchunk(int64_t N) { return (N + sa3_kmean_chunk(N) - 1) / sa3_kmean_chunk(N); }
static inline int64_t sa3_quant_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d)
{ return B * H * sa3_kmean_nchunk(N) * d * 8; }

/*
 * sa3_quantize_qkv -- K smoothing plus FP4 microscaling of Q, K and V.
 *
 * Steps ("SageAttention" summary, "Approach"; "SageAttention3" abstract):
 *   mean[bh][c] = fp32( (sum_t K[bh][t][c] in fp64) / N in fp64 )
 *   K_s = fp32(K) - mean            (one fp32 subtraction; K is not modified)
 *   for every 16-element block x of Q, K_s (along d) and V (along tokens):
 *     s = E4M3_RN_satfinite(fp32(max|x| / 6)), r = fp32(1/s),
 *     code_i = E2M1_RN_satfinite(fp32(x_i * r)), all codes 0 if s == 0.
 * Rounding is to nearest even; a negative value that rounds to zero keeps
 * its sign (code 0x8).  The fp64 sums are bit-identical to any other
 * order whenever they are exact, which holds for bf16 inputs whose
 * magnitudes span less than 2^30 at N <= 2^15.
 *
 * q, k, v    : bf16 [B][H][N][d], device, 16-byte aligned, read only.
 * out        : the seven output buffers above (device; written).
 * workspace  : device scratch of at least sa3_quant_workspace_bytes bytes
 *              (contents on entry are ignored).
 * Returns SA3_OK or an error code (see top of file).
 */
int sa3_quantize_qkv(const void *q, const void *k, const void *v,
                     int B, int H, int N, int d,
                     const sa3_qkv_fp4 *out,
                     void *workspace, size_t workspace_bytes,
                     struct CUstream_st *stream);

/*
 * sa3_attn_fwd -- O = softmax(Q^ K^T * sm_scale) V^ with FP4 P, bf16 out.
 *
 * Per (bh, 128-row Q block), for KV blocks j = 0.. (causal: j <= Q block):
 *   S = Q^ K^_j^T on the block-scaled FP4 tensor cores (fp32 accumulate);
 *   t = S * fp32(sm_scale * log2 e); columns >= N and, if causal, columns
 *   > row are -inf; m' = max(m, rowmax t); alpha = 2^(m - m');
 *   P = 2^(t - m'); l = alpha*l + rowsum(P);
 *   P^ = P microscaled per 16 columns exactly as in sa3_quantize_qkv;
 *   O = alpha*O + P^ V^_j (block-scaled FP4, fp32 accumulate); m = m'.
 * out = bf16_RN(O / l).  ("Online normalizer calculation for softmax" and
 * the FlashAttention papers, in the SageAttention3 reference list.)
 *
 * Accuracy: the recipe above is followed step by step, but not to the bit.
 * The exponentials use the hardware's approximate exp2.  1/s is folded into
 * the exponent: y = 2^(S*c + (log2(1/s) - m')) from one fused multiply-add,
 * and l is formed as sum_b s_b * sum(y).  Tensor-core sums run in their own
 * order.  So a P code may differ from the recipe's where the value sits at
 * a rounding boundary, and an output may land one bf16 ulp away where the
 * recipe's own fp32 value sits on a rounding midpoint (peaked rows, whose
 * values are short binary fractions, have many).  Rounding ties aside, the
 * outputs were measured within relative L2 1.4e-3 of the recipe in every
 * 128-row block, for softmax scales up to 1024/sqrt(d) (logits up to about
 * 10^6) on LLM- and video-DiT-shaped inputs, both masks; the parity tests
 * hold every block to 2e-3.  Scaled logits must be finite in fp32.
 *
 * in       : quantized operands from sa3_quantize_qkv for the same shape.
 * causal   : 0 or 1 (mask col > row, rows and columns both from 0).
 * sm_scale : softmax scale; <= 0 selects 1/sqrt(d).
 * out      : bf16 [B][H][N][d], device, 16-byte aligned (written).
 * Returns SA3_OK or an error code (see top of file).
 */
int sa3_attn_fwd(const sa3_qkv_fp4 *in, int B, int H, int N, int d,
                 int causal, float sm_scale, void *out,
                 struct CUstream_st *stream);

/*
 * sa3_quantize_qkv_lens, sa3_attn_fwd_lens -- the two calls above with a
 * query length Nq that may differ from the key/value length Nkv (cross
 * attention, decoding against a longer key/value sequence, chunked prefill).
 * The pages define the method for one sequence; these take its plainest
 * extension, used by the FlashAttention family in the same reference list:
 *
 *   q          : bf16 [B][H][Nq][d];  k, v : bf16 [B][H][Nkv][d].
 *   out / in   : q_fp4, q_sf sized with Nq (sa3_qk_fp4_bytes(B, H, Nq, d),
 *                sa3_qk_sf_bytes(B, H, Nq, d)); k_fp4, k_sf, vt_fp4, vt_sf
 *                sized with Nkv; the K mean runs over the Nkv keys;
 *                workspace: sa3_quant_workspace_bytes(B, H, Nkv, d).
 *   causal = 1 : query row r sees keys 0 .. r + Nkv - Nq (the last query is
 *                aligned with the last key; for Nq == Nkv the usual mask).
 *                A row that sees no key (r + Nkv - Nq < 0) outputs 0.
 *   out (attn) : bf16 [B][H][Nq][d].
 *
 * flags (attention): 0, or SA3_P_TWO_LEVEL -- P is scaled by 2^11 before it
 *   is microscaled (the largest power of two with 2^k / 6 <= 448, so no
 *   block scale saturates) and O / l is unchanged by it because l carries
 *   the same factor.  Being exact in binary, the pre-scale changes only the
 *   16-column blocks whose E4M3 scale would be subnormal or 0 (P below
 *   6 * 2^-6 relative to the row maximum), which then keep 3 significant
 *   scale bits.  The pages do not describe it: an accuracy option, off by
 *   default.  Other bits: SA3_ERR_INVALID_ARG.
 *
 * Everything else -- block recipe, arguments, errors, asynchrony -- is as in
 * sa3_quantize_qkv / sa3_attn_fwd, which are these calls with Nq == Nkv and
 * flags 0.  Both lengths obey the shape limits at the top of this file.
 */
#define SA3_P_TWO_LEVEL 1u
int sa3_quantize_qkv_lens(const void *q, const void *k, const void *v,
                          int B, int H, int Nq, int Nkv, int d,
                          const sa3_qkv_fp4 *out,
                          void *workspace, size_t workspace_bytes,
                          struct CUstream_st *stream);
int sa3_attn_fwd_lens(const sa3_qkv_fp4 *in, int B, int H, int Nq, int Nkv, int d,
                      int causal, float sm_scale, unsigned int flags, void *out,
                      struct CUstream_st *stream);

/*
 * sa3_quantize_qkv_ex, sa3_attn_fwd_ex -- the _lens calls with option flags.
 *
 * SA3_V_SMOOTH: V is smoothed like K.  The quantizer also forms the mean of
 *   V over its Nkv tokens (fp64 sum, fp64 divide, one rounding to fp32, as
 *   for K), writes it to v_mean (fp32 [B][H][d], device, 16-byte aligned,
 *   caller-owned) and quantizes V_s = fp32(V) - mean (one fp32 subtraction;
 *   padding tokens stay 0) instead of V.  Attention, given the same v_mean,
 *   adds it back after O / l:  out = bf16(O / l + mean), in fp32 (a row that
 *   sees no key still outputs 0).  Softmax rows sum to 1, so this leaves
 *   attention unchanged in exact arithmetic -- the argument the SageAttention
 *   summary ("Approach") gives for K, applied to V's per-channel mean -- and
 *   it helps when V has a large per-channel offset.  The pages do not
 *   describe it: an accuracy option, off by default.  The quantizer's
 *   workspace doubles (V's partial sums): sa3_quant_workspace_bytes_ex.
 *   V smoothing needs V's mean before V can be quantized, so V is read
 *   twice (once for the sums, once to quantize).
 * SA3_P_TWO_LEVEL (attention only): as in sa3_attn_fwd_lens.
 * SA3_SKIP_Q (quantizer) / SA3_Q_ON_LOAD (attention): Q is not quantized by
 *   the quantizer (q, out->q_fp4 and out->q_sf may be NULL and are not
 *   touched) and the attention kernel reads the bf16 Q itself (argument q:
 *   bf16 [B][H][Nq][d], device, 16-byte aligned; in->q_fp4 and in->q_sf
 *   are ignored), quantizing each 128-row tile with the same block recipe
 *   -- bit for bit the codes and scales sa3_quantize_qkv would write --
 *   before its first S.  This saves the quantizer's Q pass (Q's bf16 read,
 *   its code and scale writes and their re-read) at the cost of Q's bf16
 *   read inside the attention kernel.  The pages call the method
 *   "plug-and-play"; this is the same computation with one HBM round trip
 *   fewer.  Output identical to the two-pass path.
 *
 * v_mean is ignored (may be NULL) without SA3_V_SMOOTH, q without
 * SA3_Q_ON_LOAD.  Any other flag bit: SA3_ERR_INVALID_ARG.  Everything else
 * as in the _lens calls, which are these with flags 0 (quantizer) or flags
 * of SA3_P_TWO_LEVEL only (attention).
 */
#define SA3_V_SMOOTH 2u
#define SA3_SKIP_Q 4u
#define SA3_Q_ON_LOAD 8u
static inline int64_t sa3_quant_workspace_bytes_ex(int64_t B, int64_t H, int64_t N, int64_t d, unsigned int flags)
{ return sa3_quant_workspace_bytes(B, H, N, d) * ((flags & SA3_V_SMOOTH) ? 2 : 1); }
int sa3_quantize_qkv_ex(const void *q, const void *k, const void *v,
                        int B, int H, int Nq, int Nkv, int d, unsigned int flags,
                        const sa3_qkv_fp4 *out, float *v_mean,
                        void *workspace, size_t workspace_bytes,
                        struct CUstream_st *stream);
int sa3_attn_fwd_ex(const sa3_qkv_fp4 *in, const void *q, const float *v_mean,
                    int B, int H, int Nq, int Nkv, int d, int causal, float sm_scale,
                    unsigned int flags, void *out, struct CUstream_st *stream);

/*
 * 8-bit variant ("SageAttention: Accurate 8-Bit Attention for Plug-and-play
 * Inference Acceleration", summary, "Approach"): Q and K quantized to INT8
 * with per-block scales after K smoothing, P and V kept in FP16.  Blocks are
 * the 128-token tiles of the FP4 path, taken over all d channels:
 *   s = fp32(amax / 127), r = fp32(1 / s),
 *   code = clamp(round_half_even(fp32(x * r)), -127, 127), all 0 if s == 0;
 * V is converted to FP16 (nearest even).  Attention: S = integer dot of the
 * codes (exact, int32 on the tensor cores), t = fp32(S) * fp32(fp32(s_q *
 * s_k) * sm_scale * log2 e), the online softmax of sa3_attn_fwd, P
 * converted to FP16, O += P V in fp32, out = bf16(O / l).  Lengths, masks
 * and the empty-row rule as in sa3_attn_fwd_lens.  No E4M3 block scales.
 *
 *   q_i8     int8 [B*H][N_p(Nq)][d]       q_scale  fp32 [B*H][N_p(Nq)/128]
 *   k_i8     int8 [B*H][N_p(Nkv)][d]      k_scale  fp32 [B*H][N_p(Nkv)/128]
 *   vt_f16   fp16 [B*H][d][N_p(Nkv)]      k_mean   fp32 [B*H][d]
 * Padding tokens: code 0, fp16 0.  All device pointers, 16-byte aligned.
 */
typedef struct sa3_qkv_i8 {
    void *q_i8;
    float *q_scale;
    void *k_i8;
    float *k_scale;
    void *vt_f16;
    float *k_mean;
} sa3_qkv_i8;
static inline int64_t sa3_i8_bytes(int64_t B, int64_t H, int64_t N, int64_t d)
{ return B * H * sa3_padded_len(N) * d; }
static inline int64_t sa3_i8_scale_bytes(int64_t B, int64_t H, int64_t N)
{ return B * H * (sa3_padded_len(N) / 128) * 4; }
static inline int64_t sa3_vt_f16_bytes(int64_t B, int64_t H, int64_t N, int64_t d)
{ return B * H * d * sa3_padded_len(N) * 2; }

/* workspace: sa3_quant_workspace_bytes(B, H, Nkv, d), as for the FP4 path. */
int sa3_quantize_qkv_i8(const void *q, const void *k, const void *v,
                        int B, int H, int Nq, int Nkv, int d,
                        const sa3_qkv_i8 *out,
                        void *workspace, size_t workspace_bytes,
                        struct CUstream_st *stream);
int sa3_attn_fwd_i8(const sa3_qkv_i8 *in, int B, int H, int Nq, int Nkv, int d,
                    int causal, float sm_scale, void *out,
                    struct CUstream_st *stream);

/*
 * sa3_attn_fwd_i8_lse -- the 8-bit forward as used for training
 * ("SageAttention3: Microscaling FP4 Attention for Inference and An
 * Exploration of 8-Bit Training", abstract: 8-bit attention in both the
 * forward and the backward pass).  The backward pass needs each row's
 * softmax normaliser to rebuild P; this call is sa3_attn_fwd_i8 that also
 * writes it:
 *
 *   lse : fp32 [B][H][Nq], device, 4-byte aligned, caller-owned.
 *         lse[r] = ln 2 * (m + log2 l), m the row's final running maximum
 *         of t (base-2 units, t as above) and l its fp32 row sum of P, so
 *         lse = ln sum_j exp(sm_scale * s_q s_k * S_rj) over the keys the
 *         row sees, up to fp32 rounding.  A row that sees no key gets +inf
 *         (its P = exp(s - lse) is then 0).
 *
 * lse == NULL is sa3_attn_fwd_i8.  A misaligned lse: SA3_ERR_INVALID_ARG.
 * Other arguments, errors and asynchrony as in sa3_attn_fwd_i8.
 */
int sa3_attn_fwd_i8_lse(const sa3_qkv_i8 *in, int B, int H, int Nq, int Nkv, int d,
                        int causal, float sm_scale, void *out, float *lse,
                        struct CUstream_st *stream);

/*
 * sa3_quantize_qkv_noalloc -- sa3_quantize_qkv without a caller workspace.
 *
 * There is no counterpart in the paper: this is a convenience for callers
 * that cannot hand the library device memory at call time, for instance a
 * plug-in layer inside a framework that owns every device allocation and
 * exposes no allocator to plug-ins, or a latency-critical path where a
 * cudaMalloc (which may synchronize the device) is not acceptable.
 *
 * Same arguments, outputs and results as sa3_quantize_qkv, minus the
 * workspace: the K-mean partial sums go to a fixed scratch array that the
 * library holds in device memory on every GPU that loads it, until the
 * process exits.  The array holds SA3_NOALLOC_SCRATCH_BYTES bytes, so the
 * call accepts shapes with sa3_quant_workspace_bytes(B, H, N, d) <=
 * SA3_NOALLOC_SCRATCH_BYTES (at most 16 chunks, so B*H*d <= 32768) and
 * returns SA3_ERR_UNSUPPORTED otherwise.
 * It calls no allocation routine.
 *
 * The first call on a device looks up that device's copy of the array
 * (cudaGetSymbolAddress, with the device current) and keeps the address
 * for the life of the process; make that first call outside any stream
 * capture.  The address belongs to the device's primary context, the one
 * the CUDA runtime and PyTorch use: call this from that context only, and
 * not after cudaDeviceReset (the kept address is then stale).  All calls share the one array: two calls
 * whose kernels overlap on the GPU (different streams without ordering)
 * race on it and give undefined results.  Nothing in the array needs to
 * start at zero -- every call rewrites all the scratch it reads -- and it
 * keeps the last call's contents.
 */
#define SA3_NOALLOC_SCRATCH_BYTES (4u << 20)
int sa3_quantize_qkv_noalloc(const void *q, const void *k, const void *v,
                             int B, int H, int N, int d,
                             const sa3_qkv_fp4 *out,
                             struct CUstream_st *stream);

/*
 * sa3_device_status -- synchronizes `stream`, returns SA3_ERR_TIMEOUT if
 * a kernel of this library gave up on a bounded wait since the last call
 * (and clears the record), SA3_ERR_CUDA if the stream reports an error,
 * else SA3_OK.
 */
int sa3_device_status(struct CUstream_st *stream);

/*
 * sa3_selftest_wait_timeout -- exercises the failure path of the bounded
 * device waits: enqueues one warp that waits, through the same routine the
 * kernels above use, on a barrier nothing arrives on, for `limit_us`
 * microseconds (1 .. 10^7).  The wait gives up, records SA3_ERR_TIMEOUT in
 * the status word and the kernel returns; the CUDA context stays usable.
 * A following sa3_device_status() returns SA3_ERR_TIMEOUT (and clears it).
 * No counterpart in the method; for tests of failure detection.
 */
int sa3_selftest_wait_timeout(unsigned int limit_us, struct CUstream_st *stream);

/*
 * sa3_probe_fp4_mma -- measures the block-scaled FP4 tensor-core rate that
 * bounds sa3_attn_fwd.  No counterpart in the method: a measurement aid for
 * the attention roofline.  Enqueues `ctas` CTAs (one per SM when ctas is
 * the SM count; each claims enough shared memory to be alone on its SM),
 * each issuing `iters` (1 .. 2^18) tcgen05.mma.kind::mxf4nvf4 block-scaled
 * MMAs of M = 128, N = n (128 or 256), K = 64 from shared memory into one
 * TMEM accumulator: 2 * 128 * n * 64 operations each.  All codes are E2M1
 * 1.0 and all scales E4M3 1.0, so every accumulator element ends at
 * exactly 64 * iters.  out: device fp32 [2 * ctas], 4-byte aligned; CTA c
 * writes the smallest element of accumulator column 0 to out[2c] and the
 * largest of column n-1 to out[2c+1] (both 64 * iters when the tensor core
 * did the work).  The caller times the launch (CUDA events on `stream`).
 * Bad arguments: SA3_ERR_INVALID_ARG; launch failure: SA3_ERR_CUDA.
 */
int sa3_probe_fp4_mma(int ctas, int n, int iters, float *out, struct CUstream_st *stream);

/* Library version string, e.g. "libsa3 0.1.0 (sm_100a)". Host memory,
 * static, never freed. */
const char *sa3_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SA3_H */
