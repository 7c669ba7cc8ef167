/*
 * hifa4.h - C ABI of the B200 (sm_100a) 4-bit FlashAttention forward.
 *
 * The method is the HiFA4 operator described in "HiFA4: Training-Free 4-bit
 * FlashAttention on Ascend HIF4 NPUs for LLM Inference" (abstract; the same
 * text is printed on the scholarfeed, hf.space, thelatestinai, fugumt and
 * mlsanity pages): both QK^T and PV run as 4-bit GEMMs, the online-softmax
 * state stays in a wider float format, Smooth-QK rescales Q and K per channel
 * with calibration-static factors after RoPE, and P-Reordering accumulates the
 * softmax normalizer from the same quantized probabilities that feed PV.
 * The 4-bit format here is E2M1 elements with one E4M3 scale per 16 elements
 * along the contraction dimension (D for Q and K, tokens for V), rounded to
 * nearest even; the abstract names the Ascend HIF4 format, whose encoding it
 * does not give.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    never allocates, frees or synchronises device memory (hifa4_get_status is
 *    the only call that waits on the stream).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *  - Arguments are validated on the host before anything is launched; a
 *    violation returns HIFA4_ERR_INVALID_ARG or HIFA4_ERR_UNSUPPORTED and
 *    launches nothing. A launch failure returns HIFA4_ERR_CUDA.
 *  - Every pointer must be 16-byte aligned.
 *  - Tensors are contiguous, row-major, with the shapes given below.
 *  - Q is [B, Hq, Nq, D]; K and V are [B, Hkv, Nkv, D]. GQA: q head h reads
 *    kv head h / (Hq / Hkv).
 *  - Supported: D in {64, 128, 256}; Hq % Hkv == 0; Nkv % 128 == 0;
 *    Nq % 16 == 0; causal needs Nq <= Nkv (bottom-right aligned: key j is
 *    visible to query i iff j <= i + Nkv - Nq).
 */
#ifndef HIFA4_H
#define HIFA4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hifa4_stream_t;   /* same type as cudaStream_t */

typedef enum {
    HIFA4_OK = 0,
    HIFA4_ERR_INVALID_ARG = 1,   /* bad pointer, shape, alignment or value */
    HIFA4_ERR_UNSUPPORTED = 2,   /* valid request outside what the kernels cover */
    HIFA4_ERR_CUDA = 3,          /* a CUDA call or launch failed */
    HIFA4_ERR_TIMEOUT = 4        /* a bounded wait inside a kernel expired */
} hifa4_status;

/* Normalizer modes of the attention kernel (HiFA4 abstract, P-Reordering):
 * P_REORDER            l accumulated from the quantized P_hat that feeds the
 *                      PV GEMM, fused into that GEMM as an extra V column of ones.
 * HIGH_PRECISION_L     l accumulated from the unquantized fp32 P (the
 *                      "higher-precision reconstruction" the abstract compares with). */
typedef enum { HIFA4_NORM_P_REORDER = 0, HIFA4_NORM_HIGH_PRECISION_L = 1 } hifa4_norm_mode;

typedef enum { HIFA4_F16 = 0, HIFA4_BF16 = 1, HIFA4_F32 = 2 } hifa4_dtype;

/* Flags of the attention calls.
 * HIFA4_CAUSAL    bottom-right aligned causal mask.
 * HIFA4_SPLIT_KV  inference option (flash-decoding): the kernels may cut the
 *                 kv tiles into hifa4_attention_splits() contiguous ranges, run
 *                 the online softmax of each range from its own start (its own
 *                 running max, so P_hat is taken relative to the range's max),
 *                 and merge the ranges with their log-sum-exp weights:
 *                 O = sum_r 2^(mc_r - M) O_acc_r / sum_r 2^(mc_r - M) l_r,
 *                 M = max mc_r, LSE = M ln 2 + ln(sum_r 2^(mc_r - M) l_r).
 *                 With one range this is the plain pass. */
enum { HIFA4_CAUSAL = 1u << 0, HIFA4_SPLIT_KV = 1u << 1 };

/* Quantized operands. Layouts (u8 everywhere; codes hold two E2M1 elements
 * per byte, element 2i in the low nibble; scales are E4M3 bytes):
 *   qc  [B, Hq, Nq, D/2]         Q codes, row-major
 *   kc  [B, Hkv, Nkv, D/2]       K codes, row-major
 *   vtc [B, Hkv, Nkv/128, D, 64] V codes, transposed and tiled: each 128-token
 *                                tile of V^T is one contiguous block, channel d's
 *                                64 bytes (tokens 128j..128j+127) at row d
 *   qs, ks, vts                  scales in the MMA-ready layout below
 * MMA-ready scale layout: 512-byte atoms, each holding the scales of 128 rows x
 * 64 contraction elements (4 scales per row); row r, scale k (0..3) of an atom
 * sits at byte 16*(r%32) + 4*(r/32) + k.
 *   qs: atoms ordered [B, Hkv, Tq, D/64], Tq = ceil(G*Nq/128), G = Hq/Hkv. The
 *       rows of atom (b, g, t) are the query rows p = 128*t + r of the group's
 *       heads stacked head after head, p = (h % G)*Nq + i. Rows past G*Nq are 0.
 *   ks: atoms ordered [B, Hkv, Nkv/128, D/64], row r = token % 128.
 *   vts: atoms ordered [B, Hkv, Nkv/128, ceil(D/128), 2], row r = channel % 128
 *       of the 128-channel block, k = (token % 64)/16 of the 64-token half.
 *       When D = 64 the padding row 64 holds 0x38 (1.0): the scale of the
 *       normalizer column used by P-Reordering. Other padding rows are 0.
 * The canonical scale tensors Qs [B,Hq,Nq,D/16], Ks [B,Hkv,Nkv,D/16] and
 * Vts [B,Hkv,D,Nkv/16], and the canonical V codes Vtc [B,Hkv,D,Nkv/2]
 * (byte c of a channel row: Vtc[b,g,d,c] = vtc[b,g,c/64,d,c%64]), map one-to-one
 * onto these bytes. */
typedef struct {
    void* qc;
    void* qs;
    void* kc;
    void* ks;
    void* vtc;
    void* vts;
} hifa4_packed;

/* Bytes of each packed buffer, in the order qc, qs, kc, ks, vtc, vts, written
 * to out[6] (may be NULL). Returns their sum, or 0 for an unsupported shape. */
size_t hifa4_packed_bytes(int B, int Hq, int Hkv, int Nq, int Nkv, int D, size_t out[6]);

/* Number of kv ranges the attention calls use for this shape and flags: 4 when
 * HIFA4_SPLIT_KV is set, D <= 128, a group's query rows fit in half a tile
 * (Hq/Hkv * Nq <= 64: decode-style chunks) and Nkv >= 512; otherwise 1 (the
 * plain pass). Range r covers the kv tiles [T*r/n, T*(r+1)/n), T = Nkv/128.
 * Returns 0 for an unsupported shape. */
int hifa4_attention_splits(int B, int Hq, int Hkv, int Nq, int Nkv, int D, unsigned flags);

/* Bytes of the device workspace hifa4_attention_fwd needs: one status word
 * (padded to 256 bytes). The caller zeroes it once after allocating; a kernel
 * writes it only when a bounded wait expires, and hifa4_get_status clears it. */
size_t hifa4_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nkv, int D);

/* Smooth-QK calibration (HiFA4 abstract: "calibration-static per-channel
 * equivalent rescaling ... transferring quantization difficulty from K to Q").
 * For each kv head g and channel c: aQ = max |Q| over the batch, the N tokens
 * and the q heads of group g; aK = max |K| over the batch and tokens;
 * s = aK^alpha / aQ^(1-alpha) (alpha = 0.5 gives sqrt(aK/aQ), computed as
 * correctly rounded fp32 division and square root), s = 1 when aQ or aK is 0,
 * s_inv = RN(1/s). q: [B,Hq,N,D], k: [B,Hkv,N,D] in `dtype` (F16 or BF16);
 * s, s_inv: fp32 [Hkv, D], written (their previous contents are overwritten;
 * they also serve as the reduction scratch). alpha in (0, 1]. */
hifa4_status hifa4_calibrate_smooth(const void* q, const void* k, hifa4_dtype dtype,
                                    int B, int Hq, int Hkv, int N, int D, float alpha,
                                    float* s, float* s_inv, hifa4_stream_t stream);

/* Smooth and quantize Q, K and V (HiFA4 abstract: Smooth-QK "after RoPE",
 * then 4-bit QK^T and PV GEMMs). Q' = RN(Q*s[g]), K' = RN(K*s_inv[g]) in fp32
 * (s and s_inv both NULL: no smoothing). Per 16-element block along the
 * contraction dimension: sf = E4M3_rn_satfinite(amax * RN(1/6)), r = RN(1/sf)
 * (0 when sf = 0), code = E2M1_rn_satfinite(RN(x*r)). Q and K are blocked
 * along D, V along tokens (written transposed). q, k, v in `dtype`
 * (F16 or BF16); out points at caller-allocated buffers sized by
 * hifa4_packed_bytes. */
hifa4_status hifa4_quantize_qkv(const void* q, const void* k, const void* v, hifa4_dtype dtype,
                                int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                const float* s, const float* s_inv,
                                const hifa4_packed* out, hifa4_stream_t stream);

/* Quantize only K and V (a KV cache is quantized once, when it is appended).
 * Same rules and layouts as hifa4_quantize_qkv; out->qc / out->qs are ignored. */
hifa4_status hifa4_quantize_kv(const void* k, const void* v, hifa4_dtype dtype,
                               int B, int Hkv, int Nkv, int D, const float* s_inv,
                               const hifa4_packed* out, hifa4_stream_t stream);

/* The steps before quantization, each optional, applied in this order to the
 * pre-quantization fp32 values (no rounding to the storage type between them):
 *  1. RoPE (rope_cos != NULL), rotate-half pairing: channel d < D/2 pairs with
 *     d + D/2; with c = rope_cos[pos, d], s = rope_sin[pos, d] (tables fp32
 *     [n_pos, D/2]): x[d] <- RN(RN(x[d]*c) - RN(x[d+D/2]*s)),
 *     x[d+D/2] <- RN(RN(x[d+D/2]*c) + RN(x[d]*s)), each product and sum rounded
 *     to fp32 (no fused multiply-add). Applied to Q and K, never to V. The
 *     abstract applies Smooth-QK "after RoPE"; fusing the two removes a pass.
 *  2. Smooth-QK: x <- RN(x*s[g]) for Q, RN(x*s_inv[g]) for K (both NULL: off).
 *  3. Q-Mean auxiliary (q_mean != NULL; the abstract adopts it with
 *     P-Reordering on models where Smooth-QK is disabled, without defining it;
 *     this library reads it as Q smoothing by the mean): Q <- RN(Q - q_mean[b,h])
 *     before quantization, and the rank-one score term that subtraction
 *     removes, s_bias[b,h,j] = sum_d q_mean[b,h,d] * K'[b,g,j,d], is written
 *     from the keys K' as they enter quantization (after steps 1-2, before
 *     4-bit rounding), accumulated in fp32. hifa4_attention_fwd_ex adds s_bias
 *     to the scores.
 * Positions: query token i of every batch and head sits at q_pos[i] (int32
 * [Nq]); key token j at k_pos[j] (int32 [Nkv], or [n_new] for an append).
 * Positions outside [0, n_pos) are clamped into it. */
typedef struct {
    const float* s;          /* Smooth-QK factors [Hkv, D] or NULL */
    const float* s_inv;      /* their reciprocals [Hkv, D]; NULL exactly when s is NULL */
    const float* rope_cos;   /* [n_pos, D/2] fp32, or NULL (then rope_sin is NULL too) */
    const float* rope_sin;
    const int32_t* q_pos;    /* [Nq] */
    const int32_t* k_pos;    /* [Nkv] or [n_new] */
    int n_pos;
    const float* q_mean;     /* Q-Mean auxiliary [B,Hq,D] (see hifa4_q_mean) or NULL */
    float* s_bias;           /* [B,Hq,Nkv] fp32 output, required exactly when q_mean is set */
} hifa4_prequant;

/* hifa4_quantize_qkv with the steps of hifa4_prequant (pre may be NULL: none).
 * Table and bias pointers must be 16-byte aligned, positions 4-byte aligned. */
hifa4_status hifa4_quantize_qkv_ex(const void* q, const void* k, const void* v, hifa4_dtype dtype,
                                   int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                   const hifa4_prequant* pre, const hifa4_packed* out, hifa4_stream_t stream);

/* Q-Mean: q_mean[b,h,d] (fp32 [B,Hq,D]) = mean over the Nq tokens of Q after
 * RoPE and smoothing (pre: uses s, rope_cos, rope_sin, q_pos, n_pos; may be
 * NULL), summed in fp64 and rounded once to fp32 after an fp64 division. The
 * order of the fp64 additions is unspecified: results can differ from another
 * fp64 summation only when the exact mean lies within about 1e-16 (relative)
 * of an fp32 rounding boundary. */
hifa4_status hifa4_q_mean(const void* q, hifa4_dtype dtype, int B, int Hq, int Hkv, int Nq, int D,
                          const hifa4_prequant* pre, float* q_mean, hifa4_stream_t stream);

/* Quantize Q alone, e.g. a decode step's new queries against a packed KV cache
 * (HiFA4 abstract: Smooth-QK "after RoPE ... before quantization"). Rules,
 * steps and layout are those of the Q part of hifa4_quantize_qkv_ex: RoPE
 * (pre->rope_cos / rope_sin with pre->q_pos), the Smooth-QK multiply (pre->s,
 * indexed by kv head h / (Hq / Hkv)) and the Q-Mean subtraction (pre->q_mean)
 * may be set; pre->s_inv and pre->k_pos are ignored and pre->s_bias must be
 * NULL (the score bias belongs to the K pass). q: [B,Hq,Nq,D] in `dtype`.
 * Writes out->qc and out->qs (sized by hifa4_packed_bytes for these B, Hq,
 * Hkv, Nq, D and any Nkv); the other pointers of `out` are ignored. */
hifa4_status hifa4_quantize_q(const void* q, hifa4_dtype dtype, int B, int Hq, int Hkv, int Nq, int D,
                              const hifa4_prequant* pre, const hifa4_packed* out, hifa4_stream_t stream);

/* KV-cache append: quantize n_new new K and V tokens ([B, Hkv, n_new, D]) into
 * token slots [start, start + n_new) of a packed cache that holds
 * cache_tokens tokens (cache->kc, ks, vtc, vts sized by hifa4_packed_bytes
 * with Nkv = cache_tokens; qc / qs ignored). Codes and scales equal those of
 * quantizing the whole cache at once; slots outside the range are untouched.
 * Needs start % 16 == 0 and n_new % 16 == 0 (a V scale covers 16 tokens;
 * decoding keeps the last, partial 16 tokens unquantized or re-appends them),
 * start + n_new <= cache_tokens, cache_tokens % 128 == 0. pre: s_inv and RoPE
 * (k_pos has n_new entries) may be set; q_mean must be NULL. */
hifa4_status hifa4_append_kv(const void* k, const void* v, hifa4_dtype dtype, int B, int Hkv, int n_new, int D,
                             const hifa4_prequant* pre, const hifa4_packed* cache, int cache_tokens, int start,
                             hifa4_stream_t stream);

/* 4-bit attention forward (HiFA4 abstract). For each query row, one pass over
 * 128-key tiles in ascending order: S = Q_hat K_hat^T (block-scaled FP4 MMA,
 * fp32 accumulate), running max m updated every tile, c = RN(sm_scale*log2 e),
 * P = 2^(S*c - RN(m*c)), P quantized per 16 keys to P_hat with the element
 * rule above, O_acc = alpha*O_acc + P_hat V_hat (block-scaled FP4 MMA), and the
 * normalizer l per `norm` (see hifa4_norm_mode). Output O = O_acc / l in
 * `o_dtype` [B,Hq,Nq,D]; lse (fp32 [B,Hq,Nq], may be NULL) =
 * RN(m*c)*ln 2 + ln l, the natural-log log-sum-exp of sm_scale*S.
 * sm_scale: finite and > 0 (1/sqrt(D) is the usual value). flags: HIFA4_CAUSAL,
 * HIFA4_SPLIT_KV (see above).
 * workspace: hifa4_workspace_bytes() bytes, zeroed once by the caller; a
 * bounded wait that expires inside the kernel records HIFA4_ERR_TIMEOUT there
 * (read it with hifa4_get_status). Concurrent calls must use different
 * workspaces. */
hifa4_status hifa4_attention_fwd(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                 float sm_scale, unsigned flags, hifa4_norm_mode norm,
                                 void* o, hifa4_dtype o_dtype, float* lse,
                                 void* workspace, hifa4_stream_t stream);

/* Same as hifa4_attention_fwd, and also writes the quantized probabilities
 * P_hat the PV GEMM consumed: p_codes [B,Hq,Nq,Nkv/2] (two E2M1 codes per byte,
 * key 2i in the low nibble) and p_scales [B,Hq,Nq,Nkv/16] (E4M3). Tiles the
 * kernel skips (entirely above the causal diagonal for the row's 128-row
 * tile) are not written, so the caller zeroes both buffers first. A debugging
 * aid for checking P_hat against a reference; slower than the plain call. */
hifa4_status hifa4_attention_fwd_debug(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                       float sm_scale, unsigned flags, hifa4_norm_mode norm,
                                       void* o, hifa4_dtype o_dtype, float* lse,
                                       uint8_t* p_codes, uint8_t* p_scales,
                                       void* workspace, hifa4_stream_t stream);

/* Optional inputs and outputs of hifa4_attention_fwd_ex (any field may be NULL).
 *  s_bias     [B,Hq,Nkv] fp32, added to every score of head (b,h) and key j
 *             before the softmax: S = RN(Q_hat K_hat^T + s_bias) (the Q-Mean
 *             term written by hifa4_quantize_qkv_ex).
 *  p_codes    [B,Hq,Nq,Nkv/2], p_scales [B,Hq,Nq,Nkv/16]: P_hat as in
 *             hifa4_attention_fwd_debug (set both or neither).
 *  tile_sums  [B,Hq,Nq,Nkv/128,2] fp32: for each query row and 128-key tile the
 *             row visits, (sum of P_hat = codes x scales, sum of P before
 *             quantization), both relative to the row's running max at that
 *             tile. The abstract's epsilon_bar statistic is built from these
 *             (hifa4_tile_stats). Tiles a row does not visit are not written.
 * Each set field makes the call run the kernel's slower extras variant. */
typedef struct {
    const float* s_bias;
    uint8_t* p_codes;
    uint8_t* p_scales;
    float* tile_sums;
} hifa4_attention_extras;

/* hifa4_attention_fwd with the extras above (extras may be NULL: the plain call). */
hifa4_status hifa4_attention_fwd_ex(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                    float sm_scale, unsigned flags, hifa4_norm_mode norm,
                                    void* o, hifa4_dtype o_dtype, float* lse,
                                    const hifa4_attention_extras* extras, void* workspace, hifa4_stream_t stream);

/* hifa4_attention_fwd with Q given unquantized: q [B,Hq,Nq,D] in q_dtype (F16
 * or BF16) and, optionally, the Smooth-QK factors s [Hkv,D] (NULL: no
 * smoothing). The kernel quantizes each query row itself when it starts, with
 * the rule and result of hifa4_quantize_qkv (Q' = RN(Q*s), per 16 elements
 * sf = E4M3(amax * RN(1/6)), code = E2M1(RN(x * RN(1/sf)))), so O and LSE
 * equal those of hifa4_quantize_qkv + hifa4_attention_fwd bit for bit; the
 * packed Q is never written to memory. kv: the packed K and V (kc, ks, vtc,
 * vts; qc and qs are ignored), e.g. from hifa4_quantize_kv or a cache filled
 * by hifa4_append_kv. D must be 128 and the call must not select the split-kv
 * decode mode (HIFA4_ERR_UNSUPPORTED otherwise). Other arguments as for
 * hifa4_attention_fwd. */
hifa4_status hifa4_attention_fwd_q(const void* q, hifa4_dtype q_dtype, const float* s, const hifa4_packed* kv,
                                   int B, int Hq, int Hkv, int Nq, int Nkv, int D, float sm_scale, unsigned flags,
                                   hifa4_norm_mode norm, void* o, hifa4_dtype o_dtype, float* lse,
                                   void* workspace, hifa4_stream_t stream);

/* Epsilon-bar per tile (HiFA4 abstract: the net probability-mass change of
 * quantizing P, median -0.064 over the Qwen3-8B trace's tiles). A tile is 128
 * query rows (the last one of a head may be shorter) of one (b,h) x one
 * 128-key tile: eps_bar = mean over the tile's rows with sum P > 0 of
 * (sum P_hat / sum P - 1) in fp32, NaN when no row of the tile has mass.
 * tile_sums as written by hifa4_attention_fwd_ex, zeroed before that call so
 * that unvisited tiles read as empty; eps_bar fp32 [B,Hq,ceil(Nq/128),Nkv/128]. */
hifa4_status hifa4_tile_stats(const float* tile_sums, int B, int Hq, int Nq, int Nkv, float* eps_bar,
                              hifa4_stream_t stream);

/* hifa4_attention_fwd without a caller-provided workspace, for callers that
 * cannot allocate device memory: for example a plugin inside a host runtime
 * that owns all device memory and exposes no allocator, or a latency-critical
 * path that cannot afford cudaMalloc's implicit device synchronisation. It
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine);
 * its scratch is a fixed 4096-byte array in the library's device image, which
 * every GPU that loads the library holds until the process exits. (The HiFA4
 * paper has no counterpart of this call; it is an integration aid.)
 * Arguments, layouts and results are those of hifa4_attention_fwd.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, no allocation) with that device current, and so
 *    does the first call after the device's context was re-created (for
 *    example by cudaDeviceReset); make such a call before any stream capture.
 *    Devices with an ordinal of 64 or more return HIFA4_ERR_UNSUPPORTED.
 *  - Arguments are checked as for hifa4_attention_fwd before anything is
 *    queued; then every call clears the part of the array it uses (the status
 *    word) on `stream` and launches.
 *  - Problems whose hifa4_workspace_bytes exceeds 4096 return
 *    HIFA4_ERR_UNSUPPORTED without launching.
 *  - All calls on a device share the one array: calls that overlap on the GPU
 *    (different streams without ordering between them) race on it. Order them.
 *  - A bounded wait that expires in the kernel is not reported back by this
 *    call (it has no workspace to read); use hifa4_attention_fwd with a
 *    workspace when that status is needed. */
hifa4_status hifa4_attention_fwd_noalloc(const hifa4_packed* in, int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                                         float sm_scale, unsigned flags, hifa4_norm_mode norm,
                                         void* o, hifa4_dtype o_dtype, float* lse, hifa4_stream_t stream);

/* Synchronises `stream`, then returns the status a kernel recorded in
 * `workspace` (HIFA4_OK or HIFA4_ERR_TIMEOUT) or HIFA4_ERR_CUDA if the stream
 * reported an error. Clears the recorded status. It also reports (as
 * HIFA4_ERR_TIMEOUT) and clears the device-wide status word of the quantize
 * passes (hifa4_quantize_qkv*, hifa4_quantize_q, hifa4_quantize_kv,
 * hifa4_append_kv), which a
 * bounded wait for the pass's own input copies sets when it expires. */
hifa4_status hifa4_get_status(void* workspace, hifa4_stream_t stream);

/* Test hook for the timeout path: sets the wait limit (nanoseconds) that the
 * bounded waits of the attention kernel and of the quantize passes use from
 * the next launch on (0 restores the default of 2 s), and, when `stall_loads`
 * is nonzero, makes the next launches issue no loads (the attention kernel's
 * load warp, the quantize pass's Q/K row copies), so every wait on them runs
 * out with nothing in flight. Returns the previous limit. */
long long hifa4_debug_set_wait_limit(long long limit_ns, int stall_loads);

/* Description of the last CUDA error behind an HIFA4_ERR_CUDA returned to
 * the calling thread ("no error" if there was none). */
const char* hifa4_last_cuda_error(void);

/* Human-readable name of a status code. */
const char* hifa4_status_string(hifa4_status status);

/* Library version, major*10000 + minor*100 + patch. */
int hifa4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HIFA4_H */
