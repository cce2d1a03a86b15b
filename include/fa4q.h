/*
 * fa4q.h - C ABI of the fused 4-bit microscaled FlashAttention library (B200, sm_100a).
 *
 * Plain pointers and sizes only.  Unless stated otherwise every pointer is a CUDA device
 * pointer owned by the caller, 16-byte aligned, and every call is asynchronous on `stream`
 * (a cudaStream_t passed as void*; NULL = the legacy default stream).  The library keeps
 * no per-call state; its only global state is one device status word written by kernels
 * whose bounded waits expire (read it with fa4q_device_status).
 *
 * Errors: argument errors are caught on the host before any launch and return
 * FA4Q_ERR_INVALID_ARG; shapes outside the supported set return FA4Q_ERR_UNSUPPORTED;
 * a failed launch returns FA4Q_ERR_CUDA.  No call ever falls back to a CPU path.
 *
 * Formats (BitDecoding-FP4: Algorithm-System Co-Design for Native FP4 KV Cache Decoding,
 * section "The KV Cache Bottleneck in Long-Context LLM Serving"; MXAttention, Abstract):
 *   elements are E2M1 (+-{0, .5, 1, 1.5, 2, 3, 4, 6}), two per byte, element 2i in the low
 *   nibble of byte i;
 *   NVFP4: 16-element blocks, one unsigned E4M3 scale byte each, optional FP32 tensor scale g;
 *   MXFP4: 32-element blocks, one E8M0 scale byte each (2^(b-127)).
 *
 * Scale-factor layouts:
 *   FA4Q_SF_ROWMAJOR: matrix [R][C] -> bytes [R][C/blk].
 *   FA4Q_SF_TILED   : the layout the block-scaled tensor-core MMA consumes.  Rows are
 *     grouped in tiles of 128 and scale columns in groups of 4; each (row tile, group)
 *     is a 512-byte atom.  nRT = ceil(R/128), nG = ceil(C/128) * (32/blk) (the columns
 *     are padded to whole 128-element tiles).  Atom (rt, g) starts at (rt*nG + g)*512;
 *     row r, scale column k sits at byte (r%32)*16 + ((r%128)/32)*4 + (k%4) of atom
 *     (r/128, k/4).  Padding bytes hold the scale of an all-zero block (0).
 *     Size: fa4q_sf_tiled_bytes(R, C, fmt).
 */
#ifndef FA4Q_H_
#define FA4Q_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { FA4Q_NVFP4 = 0, FA4Q_MXFP4 = 1 } fa4q_format;

typedef enum {
  FA4Q_OK = 0,
  FA4Q_ERR_INVALID_ARG = 1,
  FA4Q_ERR_UNSUPPORTED = 2,
  FA4Q_ERR_CUDA = 3,
  FA4Q_ERR_TIMEOUT = 4
} fa4q_status;

typedef enum {
  FA4Q_AXIS_INNER = 0, /* blocks along the contiguous axis (Q, K: along the head dim)      */
  FA4Q_AXIS_OUTER = 1  /* blocks along rows (tokens); the output is transposed (V -> V^T)  */
} fa4q_axis;

typedef enum { FA4Q_SF_ROWMAJOR = 0, FA4Q_SF_TILED = 1 } fa4q_sf_layout;

/* Human-readable name of a status code (static string). */
const char* fa4q_status_string(fa4q_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int fa4q_version(void);

/* Bytes of a FA4Q_SF_TILED scale array for an [rows][cols] matrix. */
size_t fa4q_sf_tiled_bytes(int64_t rows, int64_t cols, fa4q_format fmt);

/*
 * fa4q_quantize - blockwise E2M1 quantisation with per-block scales.
 *
 * Source: BitDecoding-FP4, "The KV Cache Bottleneck ..." (block microscaling, E2M1
 * elements, E8M0 / E4M3 scales); MXAttention, Abstract (power-of-two scaling, scale
 * bound Qmax = 7.25); HiFA4, Abstract (Smooth-QK: a static per-channel multiplier applied
 * after RoPE, before quantisation).
 *
 * x           bf16, logically [groups][rows][cols]; element (g, r, c) at
 *             x[(g*rows + r)*row_stride + c].  row_stride >= cols, multiple of 8.
 * fmt         FA4Q_NVFP4 or FA4Q_MXFP4.
 * axis        INNER: blocks of blk consecutive columns; cols % blk == 0.
 *               packed_out [groups][rows][cols/2]; scales per `sf_layout` over the
 *               [rows][cols] matrix of each group (groups stacked, each group's tiled
 *               array is fa4q_sf_tiled_bytes(rows, cols) bytes).
 *             OUTER: blocks of blk consecutive rows of each column; output transposed.
 *               rows_pad = rows rounded up to 32 (zero tokens in the padding);
 *               packed_out [groups][cols][rows_pad/2]; scales over the [cols][rows_pad]
 *               transposed matrix of each group.
 * qmax        scale bound.  NVFP4: 0 -> 6; scale = UE4M3(amax / (qmax * g)).
 *             MXFP4: 0 -> OCP rule (e = floor(log2 amax) - 2); > 0 -> UOS rule (the
 *             smallest e with amax <= qmax * 2^e), e.g. 7.25.
 * tensor_scale  NVFP4 second-level FP32 scale g (must be > 0; 1 = none); ignored for MXFP4.
 * smooth_mul  nullable FP32 [n][cols]; row r of group g is multiplied elementwise by
 *             smooth_mul[((g % smooth_heads) / smooth_ratio)*cols + c] before the block
 *             maximum (INNER only).  Pass the Q multipliers with smooth_ratio = Hq/Hkv and
 *             the K multipliers (1/lambda) with smooth_ratio = 1; smooth_heads = heads.
 * The FP32 order of operations is fixed (product qmax*g first, IEEE division), so the
 * output is bit-identical to the reference rules.
 */
fa4q_status fa4q_quantize(const void* x, int64_t groups, int64_t rows, int64_t cols,
                          int64_t row_stride, fa4q_format fmt, fa4q_axis axis, float qmax,
                          float tensor_scale, const float* smooth_mul, int64_t smooth_heads,
                          int64_t smooth_ratio, fa4q_sf_layout sf_layout, uint8_t* packed_out,
                          uint8_t* scales_out, void* stream);

/*
 * fa4q_quantize_rotated - fa4q_quantize (AXIS_INNER) of Hadamard-rotated rows, an ablation:
 * the alternative to Smooth-QK for outlier channels of K.
 *
 * Source: BitDecoding-FP4, "Outlier-Aware Key Quantization" (an orthogonal Hadamard rotation
 * of the keys spreads channel outliers across the head dimension; the same rotation on the
 * query side leaves the scores unchanged).  The pages fix no normalisation or order.  Here
 * every row (after the optional smooth_mul multiply) is replaced by its unnormalised
 * Sylvester-order Walsh-Hadamard transform, computed in IEEE FP32 by butterflies in stages
 * h = 1, 2, ..., cols/2 ((a, b) -> (a + b, a - b)), then quantised exactly as fa4q_quantize.
 * Rotating both Q and K multiplies Q K^T by cols: pass sm_scale = 1/(cols*sqrt(cols)) to
 * fa4q_attn_fwd (an exact power-of-two change of the default).  V is not rotated.
 *
 * cols 64 or 128 (else FA4Q_ERR_UNSUPPORTED); other arguments, layouts and errors as
 * fa4q_quantize with axis = FA4Q_AXIS_INNER.
 */
fa4q_status fa4q_quantize_rotated(const void* x, int64_t groups, int64_t rows, int64_t cols,
                                  int64_t row_stride, fa4q_format fmt, float qmax,
                                  float tensor_scale, const float* smooth_mul, int64_t smooth_heads,
                                  int64_t smooth_ratio, fa4q_sf_layout sf_layout,
                                  uint8_t* packed_out, uint8_t* scales_out, void* stream);

/*
 * fa4q_quantize_qkv - the three quantisations of a prefill in one launch, bit-identical to
 *   fa4q_quantize(q, B*Hq,  S_q, d, d, fmt, INNER, qmax, g_q, mul_q, Hq,  Hq/Hkv, TILED, ...)
 *   fa4q_quantize(k, B*Hkv, S_k, d, d, fmt, INNER, qmax, g_k, mul_k, Hkv, 1,      TILED, ...)
 *   fa4q_quantize(v, B*Hkv, S_k, d, d, fmt, OUTER, qmax, g_v, NULL,  0,   0,      TILED, ...)
 * i.e. exactly the operands fa4q_attn_fwd reads.  Same sources as fa4q_quantize (block
 * quantisation of Q, K along d with the optional Smooth-QK multipliers, of V along tokens,
 * stored transposed).  The CTAs of one launch are split between the three tensors, so the
 * small K and V parts run beside Q instead of as two more launches.
 * q bf16 [B][Hq][S_q][d], k, v bf16 [B][Hkv][S_k][d] (contiguous); mul_q / mul_k nullable
 * FP32 [Hkv][d] (lambda and 1/lambda); outputs as fa4q_quantize's (tiled scales).  d in
 * {64, 128}; the NVFP4 tensor scales g_* are ignored for MXFP4.  Errors as fa4q_quantize.
 */
fa4q_status fa4q_quantize_qkv(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                              int S_q, int S_k, int d, fa4q_format fmt, float qmax, float g_q,
                              float g_k, float g_v, const float* mul_q, const float* mul_k,
                              uint8_t* q_packed, uint8_t* q_sf, uint8_t* k_packed, uint8_t* k_sf,
                              uint8_t* vt_packed, uint8_t* vt_sf, void* stream);

/*
 * fa4q_smooth_calibrate - static per-channel Smooth-QK multipliers from a calibration draw.
 *
 * Source: HiFA4, Abstract (calibration-static per-channel equivalent rescaling of Q and K
 * after RoPE, moving quantisation difficulty from K to Q); BitDecoding-FP4, "Outlier-Aware
 * Key Quantization" (static smoothing coefficients estimated during calibration).
 * Rule: r_c = max_t|K_tc| / max_{t, q-heads of the kv-head}|Q_tc| (FP32 division);
 * lambda_c = sqrt(r_c) rounded to the nearest power of two (log domain, ties up), clamped
 * to [2^-8, 2^8]; r = 0 -> 2^-8, r = inf -> 2^8, NaN -> 1.
 *
 * q_cal bf16 [Hq][T][d], k_cal bf16 [Hkv][T][d]; outputs FP32 [Hkv][d]:
 * mul_q = lambda, mul_k = 1/lambda (both exact powers of two).
 */
fa4q_status fa4q_smooth_calibrate(const void* q_cal, const void* k_cal, int Hq, int Hkv, int T,
                                  int d, float* mul_q, float* mul_k, void* stream);

/*
 * fa4q_attn_fwd - fused 4-bit prefill attention (one launch).
 *
 * Source: HiFA4, Abstract (QK^T and PV as 4-bit GEMMs under an online softmax;
 * P-Reordering: the normaliser accumulates the same quantised P_hat that feeds the PV
 * GEMM, fused into that GEMM); MXAttention, Abstract (Pre-Normalization Quantization:
 * the unnormalised exponentials are quantised before the row sum); BitDecoding-FP4,
 * "Underflow-Aware Probability Scaling" (NVFP4 P uses the static tensor scale
 * g_P = 1/(6*448)).  Key tiles are 128 wide; P blocks run along keys.
 *
 * q, q_sf     packed [B][Hq][S_q][d/2]; tiled scales, one [S_q][d] matrix per (b, h).
 * k, k_sf     packed [B][Hkv][S_k][d/2]; tiled scales per (b, kv-head).
 * vt, vt_sf   V^T packed [B][Hkv][d][S_kpad/2], S_kpad = S_k rounded up to 32 (the OUTER
 *             output of fa4q_quantize); tiled scales per (b, kv-head) over [d][S_kpad].
 * g_q,g_k,g_v NVFP4 tensor scales used when quantising (1 for MXFP4).
 * d           64 or 128.  Hq % Hkv == 0; q-head h reads kv-head h*Hkv/Hq.
 * qmax_p      MXFP4 P scale rule (0 = OCP, > 0 = UOS bound); ignored for NVFP4.
 * causal      top-left aligned (query i sees keys <= i); requires S_q == S_k.
 * sm_scale    0 -> 1/sqrt(d).
 * out         [B][Hq][S_q][d], bf16 (out_is_fp32 = 0) or fp32.
 * lse         nullable FP32 [B][Hq][S_q]: natural log-sum-exp m + ln(sum P_hat).
 */
fa4q_status fa4q_attn_fwd(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                          const uint8_t* k_sf, const uint8_t* vt, const uint8_t* vt_sf,
                          float g_q, float g_k, float g_v, int B, int Hq, int Hkv, int S_q,
                          int S_k, int d, fa4q_format fmt, float qmax_p, int causal,
                          float sm_scale, void* out, int out_is_fp32, float* lse, void* stream);

/*
 * fa4q_attn_fwd_ex - fa4q_attn_fwd with two ablations of the method (fa4q_attn_fwd is this
 * call with rescale_tau = 0 and l_from_ptilde = 0).
 *
 * 1. Conditional rescaling (rescale_tau > 0).
 * Source: the FlashAttention-4 abstract on the FLAMIA page names conditional softmax
 * rescaling among its Blackwell techniques; the pages give no rule.  Here: the reference
 * maximum m of a query row moves to a key tile's maximum only when that maximum exceeds m
 * by more than rescale_tau binades, so the unnormalised exponentials P~ = exp(s - m) reach
 * up to 2^rescale_tau and the O/l accumulators are rescaled only when m moves.  P~ is then
 * quantised exactly as before (PNQ against the reference m; the MXFP4 block exponents absorb
 * P~ > 1).  P_hat therefore differs from the exact-maximum result (the output stays a convex
 * combination of V_hat).
 *
 * rescale_tau  integer in [0, 30]; anything else -> FA4Q_ERR_INVALID_ARG.  rescale_tau > 0
 *              with NVFP4 -> FA4Q_ERR_UNSUPPORTED: a key whose score equals a kept
 *              reference gets P~ = 1, i.e. y = 1/(s g_P 2^tau), an exact E2M1 tie for some
 *              UE4M3 scales s that the kernel's exponential form cannot reproduce; with
 *              MXFP4 that value is 2^-e, formed exactly from the score difference.
 *
 * 2. The inconsistent normaliser (l_from_ptilde = 1).  Source: HiFA4, Abstract - the
 * normaliser accumulated from the unquantised exponentials while the numerator uses P_hat
 * gives a coherent output-scaling error with net mass loss, which P-Reordering removes.
 * Here the softmax threads sum P~ in FP32 (per tile, rescaled like O) and the epilogue divides
 * by that sum; the PV product is unchanged, so each output row is the P-Reordering output
 * times sum P_hat / sum P~ (the LSE, when asked for, uses the same sum).
 * l_from_ptilde  0 or 1; anything else -> FA4Q_ERR_INVALID_ARG.
 *
 * All other arguments, layouts and errors as fa4q_attn_fwd.
 */
fa4q_status fa4q_attn_fwd_ex(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                             const uint8_t* k_sf, const uint8_t* vt, const uint8_t* vt_sf,
                             float g_q, float g_k, float g_v, int B, int Hq, int Hkv, int S_q,
                             int S_k, int d, fa4q_format fmt, float qmax_p, int causal,
                             float sm_scale, int rescale_tau, int l_from_ptilde, void* out,
                             int out_is_fp32, float* lse, void* stream);

/*
 * fa4q_attn_fwd_hybrid - hybrid-precision causal prefill: window and vertical-line keys in
 * BF16, the rest in FP4, under one online softmax, in one kernel.
 *
 * Source: HyQuant (Hybrid-Precision Quantization for LLM Attention): the keys of each query
 * are split into vertical-line positions, a recent sliding window and the 4-bit remainder;
 * vertical lines and the window stay in FP16/BF16; low-bit and full-precision GEMMs share
 * one FlashAttention-style kernel and one online softmax.  Reading (the pages give no order
 * or masks): query row i takes the window {j : i - window < j <= i} and the vertical lines
 * {v : v <= i - window} from the BF16 inputs first (unquantised P), then the FP4 key tiles
 * (width 128, in order) with the keys of those two classes masked out, pre-normalisation
 * quantisation of P against the running maximum that started from the BF16 part, and the
 * normaliser from P_hat; every visible key counts once.  The kernel runs the BF16 part as
 * tensor-core tiles of 64 keys (window band, then vertical lines) ahead of the FP4 tiles of
 * each 128-row query tile; the BF16 probabilities enter their PV products rounded to bf16.
 *
 * q, q_sf, k, k_sf, vt, vt_sf  FP4 operands as for fa4q_attn_fwd (S_q = S_k = S), quantised
 *             from Q, K, V with the vertical-line rows of K and V zeroed first (as the decode
 *             cache; the window keys keep their FP4 copies, later rows read them).
 * q_bf16, k_bf16, v_bf16  bf16 [B][H][S][d] (H = Hq for q, Hkv for k, v).
 * vl_pos      int32 [B][Hkv][max_vl] vertical-line positions, ascending; vl_count int32
 *             [B][Hkv] (<= max_vl); vl_k, vl_v bf16 [B][Hkv][max_vl][d] their K / V rows
 *             (rows past vl_count must hold finite values, e.g. zeros); vl_excl uint64
 *             [B][Hkv][ceil(S/64)] their bit mask (bit p%64 of word p/64).
 *             max_vl = 0: no vertical lines (the pointers may be null).
 * window      >= 1 (128 in the pages' study).  d = 128 (else FA4Q_ERR_UNSUPPORTED).
 * g_v         (NVFP4) must be a bf16 value (the BF16 part's normaliser is formed with it in
 *             bf16), else FA4Q_ERR_UNSUPPORTED.
 * Other arguments, layouts and errors as fa4q_attn_fwd (causal implied).  No workspace.
 */
fa4q_status fa4q_attn_fwd_hybrid(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                 const uint8_t* k_sf, const uint8_t* vt, const uint8_t* vt_sf,
                                 const void* q_bf16, const void* k_bf16, const void* v_bf16,
                                 const int32_t* vl_pos, const int32_t* vl_count, const void* vl_k,
                                 const void* vl_v, int max_vl, const uint64_t* vl_excl, float g_q,
                                 float g_k, float g_v, int B, int Hq, int Hkv, int S, int d,
                                 int window, fa4q_format fmt, float qmax_p, float sm_scale,
                                 void* out, int out_is_fp32, float* lse, void* stream);

/*
 * Paged FP4 KV cache (BitDecoding-FP4, "System-Level Optimization": fixed-size token
 * blocks mapped to physical memory through a block table).  Page size 64 tokens.
 * For physical page p and kv-head h:
 *   k_pages  [P][Hkv][64][d/2]      K rows, blocks along d
 *   k_sf     [P][Hkv][64][d/blk]    row-major scales
 *   vt_pages [P][Hkv][d][32]        V^T rows (64 tokens), blocks along tokens
 *   vt_sf    [P][Hkv][d][64/blk]
 * block_table [B][max_pages] int32 maps logical page j of sequence b to a physical page.
 * fp4_len [B] int32: positions [0, fp4_len[b]) of sequence b live in the FP4 pages.
 * excl_mask nullable uint64 [B][Hkv][max_pages]: bit t of word j marks position 64*j + t
 *   as held in the full-precision set instead (its FP4 slot is zero and is skipped).
 */

/*
 * fa4q_quantize_kv_pages - quantise K and V of positions [0, fp4_len[b]) into the paged
 * FP4 cache, zero-filling excluded slots before quantisation.
 * Source: HyQuant (Hybrid-Precision Quantization for LLM Attention): the KV cache is
 * stored in the hybrid way, vertical-line tokens in full precision, the rest in 4 bits.
 *
 * k, v bf16 [B][Hkv][L][d] (contiguous; L >= max fp4_len).  Writes only the pages that
 * block_table maps for j < ceil(fp4_len[b]/64); slots >= fp4_len in the last page are zero.
 */
fa4q_status fa4q_quantize_kv_pages(const void* k, const void* v, int B, int Hkv, int L, int d,
                                   const int32_t* fp4_len, const uint64_t* excl_mask,
                                   const int32_t* block_table, int max_pages, fa4q_format fmt,
                                   float g_k, float g_v, uint8_t* k_pages, uint8_t* k_sf,
                                   uint8_t* vt_pages, uint8_t* vt_sf, void* stream);

/* Workspace bytes fa4q_decode needs for `num_splits` (0 = the automatic choice). */
size_t fa4q_decode_workspace_size(int B, int Hq, int Hkv, int d, int max_pages, int num_splits);

/*
 * fa4q_decode - one query token per sequence over the hybrid cache: FP4 paged remainder
 * (dequantised inside the scan), a BF16 vertical-line set and a BF16 window, under one
 * softmax; split-K over pages with a combine of the (m, l, o) partials.
 * Source: HyQuant (vertical-line + window tokens in full precision, fused-dequant decode
 * scan, no full-precision cache materialised); BitDecoding-FP4, "System-Level
 * Optimization" (paged cache, block table).
 *
 * q        bf16 [B][Hq][d]; out bf16 [B][Hq][d].  d == 128, Hq % Hkv == 0, Hq/Hkv <= 8.
 * hp_k, hp_v  nullable bf16 [B][Hkv][max_hp][d]; hp_count int32 [B][Hkv] (<= max_hp).
 * win_k, win_v nullable bf16 [B][Hkv][W][d]; win_len int32 [B] (<= W).
 * fmt      format of the pages, as written by fa4q_quantize_kv_pages: NVFP4 (K scales
 *          [P][Hkv][64][8], V^T scales [P][Hkv][d][4]) or MXFP4 ([P][Hkv][64][4], [P][Hkv][d][2]).
 * g_k, g_v NVFP4 tensor scales of the pages (ignored for MXFP4).  sm_scale 0 -> 1/sqrt(d).
 * workspace  device scratch of fa4q_decode_workspace_size bytes (caller-owned).
 * Numerics: dequantised page values, q, the probabilities and the BF16 rows enter FP16
 * tensor-core tiles (FP32 accumulation).  FP4 page values are exact there for any scale
 * (MXFP4 block exponents are applied in FP32); q and the BF16 rows must lie within FP16's
 * range (|x| <= 65504; magnitudes below 2^-14 lose precision).
 */
fa4q_status fa4q_decode(const void* q, const uint8_t* k_pages, const uint8_t* k_sf,
                        const uint8_t* vt_pages, const uint8_t* vt_sf,
                        const int32_t* block_table, const int32_t* fp4_len,
                        const uint64_t* excl_mask, const void* hp_k, const void* hp_v,
                        const int32_t* hp_count, const void* win_k, const void* win_v,
                        const int32_t* win_len, int B, int Hq, int Hkv, int d, int max_pages,
                        int max_hp, int W, fa4q_format fmt, float g_k, float g_v,
                        float sm_scale, void* out, void* workspace, size_t workspace_bytes,
                        int num_splits, void* stream);

/*
 * fa4q_decode_fp4q - decode with FP4 tensor-core products on both sides over an all-FP4
 * paged cache: a dual-residual NVFP4 query, and the probabilities quantised before PV.
 *
 * Source: BitDecoding-FP4, "Error Sources" (the query as the sum of two FP4 tensors, the
 * second quantising the residual of the first, keeps the logits close) and "System-Level
 * Optimization" (the softmax transposed so that P is quantised inside its reduction; query
 * MMAs stacked over the paged cache).  Reading: q1 = NVFP4(q), r = q - deq(q1) in FP32,
 * q2 = NVFP4(r); scores = (deq(q1) + deq(q2)) . k_hat; the keys of a sequence are scanned in
 * tiles of 128 positions (page pairs, in position order) with pre-normalisation quantisation
 * of P against the running maximum (NVFP4, g_P = 1/(6*448)) and the normaliser from P_hat,
 * as the prefill; the scan of each sequence is cut into ranges of T = tiles_per_split whole
 * tiles (0 -> 32 tiles = 4096 keys), positions [0, 128 T), [128 T, 256 T), ...; each range
 * restarts the running state and the ranges merge exactly (log-sum-exp), so T is
 * part of the result.  The GQA heads of a kv-head share one MMA operand: the kernel computes
 * S^T = K_hat [Q_hat1 ; Q_hat2]^T and O^T += V_hat^T P_hat^T with the keys and channels on
 * the MMA's M side and the heads on N, so the result is the definition's up to FP32
 * summation order.
 *
 * q           bf16 [B][Hq][d]; out bf16 [B][Hq][d].  d = 128, Hq % Hkv == 0; Hq / Hkv > 16
 *             -> FA4Q_ERR_UNSUPPORTED.
 * k_pages ... the NVFP4 paged cache of fa4q_quantize_kv_pages (every position 0..fp4_len-1
 *             in FP4; no vertical-line set or window here); n_phys_pages = its page count.
 * g_k, g_v    NVFP4 tensor scales of the pages.  sm_scale 0 -> 1/sqrt(d).
 * workspace   device, >= fa4q_decode_fp4q_workspace_size(...) bytes, 16-byte aligned: the
 *             query tiles and the split partials.
 * MXFP4 pages -> FA4Q_ERR_UNSUPPORTED.  Other errors as fa4q_decode.  Three launches
 * (query tiles, the tcgen05 scan, the combine), asynchronous on `stream`.
 */
size_t fa4q_decode_fp4q_workspace_size(int B, int Hq, int Hkv, int d, int max_pages, int tiles_per_split);
fa4q_status fa4q_decode_fp4q(const void* q, const uint8_t* k_pages, const uint8_t* k_sf,
                             const uint8_t* vt_pages, const uint8_t* vt_sf, const int32_t* block_table,
                             const int32_t* fp4_len, int n_phys_pages, int B, int Hq, int Hkv, int d,
                             int max_pages, fa4q_format fmt, float g_k, float g_v, float sm_scale,
                             void* out, void* workspace, size_t workspace_bytes, int tiles_per_split,
                             void* stream);

/*
 * fa4q_decode_noalloc - fa4q_decode for callers that cannot allocate device memory.
 *
 * The paper has no counterpart to this call; it is a deployment convenience.  Some callers
 * cannot call cudaMalloc or hand the library a workspace: a plug-in whose host framework
 * owns every byte of device memory and gives extensions no allocator, or a latency-critical
 * serving loop where an allocation (which may synchronise the device) is not acceptable.
 * This call takes the same inputs and output as fa4q_decode but no workspace: the split
 * partials go to one static device array of 8 MiB inside the library, which every GPU that
 * loads the library holds until the process exits.  Nothing is allocated per call.
 *
 * Limit: the partials take B*Hq*(d+2)*4 bytes per split.  With num_splits = 0 the split
 * count is the automatic one, lowered as needed to fit 8 MiB; a request that does not fit
 * even with one split, or an explicit num_splits that does not fit, returns
 * FA4Q_ERR_UNSUPPORTED (use fa4q_decode with a caller workspace instead).
 * The first call on each device looks up the array's device address (with that device
 * current) and caches it; make that first call before any stream capture.
 * All calls share the array and it keeps the last call's contents (every partial is
 * rewritten before it is read, so nothing needs clearing); calls whose execution overlaps
 * on the GPU (different streams, or different host threads) race on it and must be
 * serialised by the caller.
 */
fa4q_status fa4q_decode_noalloc(const void* q, const uint8_t* k_pages, const uint8_t* k_sf,
                                const uint8_t* vt_pages, const uint8_t* vt_sf,
                                const int32_t* block_table, const int32_t* fp4_len,
                                const uint64_t* excl_mask, const void* hp_k, const void* hp_v,
                                const int32_t* hp_count, const void* win_k, const void* win_v,
                                const int32_t* win_len, int B, int Hq, int Hkv, int d,
                                int max_pages, int max_hp, int W, fa4q_format fmt, float g_k,
                                float g_v, float sm_scale, void* out, int num_splits,
                                void* stream);

/*
 * fa4q_select_vertical_lines - identify the full-precision ("vertical line") tokens of the
 * hybrid cache by accumulated column mass, and write everything the cache and the decode
 * need about them.
 * Source: HyQuant (Hybrid-Precision Quantization for LLM Attention): tokens that receive a
 * large accumulated attention mass from later queries stay in full precision (the top 5%
 * of the non-window prefix by default), the rest is stored in 4 bits; the mass comes from a
 * set of observation queries.
 *
 * Per (sequence b, kv-head h), over the candidate prefix [0, n_prefix[b]) (clamped to L):
 *   s_ij = (q_i . k_j) * sm_scale for the R = (Hq/Hkv) * n_obs observation rows q_i of the
 *          group's q-heads (row g * n_obs + t = observation t of q-head h*Hq/Hkv + g)
 *   mass_j = sum_i softmax_j(s_ij)            exact softmax over the whole prefix
 *   kept   = the ceil(rho * n_prefix[b]) largest masses, equal masses lowest position first
 *
 * q_obs      bf16 [B][Hq][n_obs][d]; R must be a multiple of 32 and at most 256.
 * k, v       bf16 [B][Hkv][L][d] (v may be null when hp_v is null).
 * n_prefix   device int32 [B].
 * rho        (0, 1], double (the count ceil(rho * n) is taken in double precision, less
 *            1e-9, so 0.05 * 32640 gives 1632); sm_scale 0 -> 1/sqrt(d).  d in {64, 128}.
 * mass       out, FP32 [B][Hkv][L] (0 outside the prefix).
 * positions  out, int32 [B][Hkv][max_select], the kept positions ascending (entries past
 *            counts[b][h] are not written); counts out, int32 [B][Hkv].
 *            max_select >= ceil(rho * L).
 * excl_mask  nullable out, uint64 [B][Hkv][max_pages] in the paged-cache layout (bit t of
 *            word j = position 64 j + t is kept); max_pages * 64 >= L.  Pass it to
 *            fa4q_quantize_kv_pages and fa4q_decode.
 * hp_k, hp_v nullable out, bf16 [B][Hkv][max_select][d]: the kept rows of k and v in
 *            position order (the decode's full-precision set; rows past counts not written).
 * workspace  device, >= fa4q_vlines_workspace_size(B, Hq, Hkv, n_obs, L) bytes, 16-byte
 *            aligned.
 * The candidates of one (sequence, kv-head) are selected in shared memory: L up to ~55,000
 * keys (4 L + 4 max_select + 8 max_pages bytes <= 227 KB), else FA4Q_ERR_UNSUPPORTED.
 * Errors: null required pointers, bad sizes, short workspace or misaligned (16-byte) bf16
 * pointers or workspace -> FA4Q_ERR_INVALID_ARG.  A device wait that expires sets the
 * status fa4q_device_status reports.  Asynchronous on `stream`.
 */
size_t fa4q_vlines_workspace_size(int B, int Hq, int Hkv, int n_obs, int L);
fa4q_status fa4q_select_vertical_lines(const void* q_obs, const void* k, const void* v,
                                       const int32_t* n_prefix, int B, int Hq, int Hkv, int n_obs,
                                       int L, int d, double rho, float sm_scale, float* mass,
                                       int32_t* positions, int32_t* counts, int max_select,
                                       uint64_t* excl_mask, int max_pages, void* hp_k, void* hp_v,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa4q_selftest_block_mma - diagnostic: one 128 x N x K block-scaled FP4 tensor-core
 * product D = A * B^T (FP32), the same MMA path the prefill kernel uses.
 * a packed [128][K/2], b packed [N][K/2] (K-major), a_sf / b_sf FA4Q_SF_TILED over
 * [128][K] and [N][K]; d_out FP32 [128][N].  K in {64, 128}; N in {16, 32, ..., 256}.
 */
fa4q_status fa4q_selftest_block_mma(const uint8_t* a, const uint8_t* a_sf, const uint8_t* b,
                                    const uint8_t* b_sf, int N, int K, fa4q_format fmt,
                                    float* d_out, void* stream);

/*
 * fa4q_selftest_bf16_mma - diagnostic: one 128 x N x K BF16 tensor-core product D = A * B
 * (FP32), through the operand layouts of the full-precision tiles of the hybrid prefill
 * (HyQuant: vertical-line and window keys in BF16): A bf16 [128][K] K-major; B bf16 [N][K]
 * (b_mn_major = 0, D = A B^T) or [K][N] (b_mn_major = 1, D = A B); both staged as 128-byte
 * swizzled 64-element column chunks.  d_out FP32 [128][N].  K in {64, 128}; N in {16, 64,
 * 128} (K-major B) or {64, 128} (MN-major B).  Synchronous errors as fa4q_attn_fwd.
 */
fa4q_status fa4q_selftest_bf16_mma(const void* a, const void* b, int N, int K, int b_mn_major,
                                   float* d_out, void* stream);

/*
 * fa4q_selftest_exp2 - diagnostic: y[i] = 2^x[i] through the FMA-pipe polynomial that the
 * prefill kernel uses for part of the unnormalised exponentials P~ = exp(S - m).  Source:
 * FLAMIA (FLAsh MIcroscaling Attention ... on Blackwell), Abstract - its FlashAttention-4
 * account lists a software-emulated exponential among the ways to relieve the exponential
 * units on B200; written here as range reduction plus a cubic minimax fit of 2^f on [0, 1)
 * (coefficients from fit_exp2_poly.py).  Relative error <= 1.6e-4 for x in [-126, 128);
 * inputs below -126 (and -inf) give a non-negative value below 2^-126.  x, y: device FP32 arrays of n
 * elements (caller-owned; n even).  Returns FA4Q_ERR_INVALID_ARG for null pointers or odd n.
 */
fa4q_status fa4q_selftest_exp2(const float* x, float* y, int64_t n, void* stream);

/*
 * fa4q_device_status - synchronise `stream`, then read and clear the device status word.
 * Returns FA4Q_ERR_TIMEOUT if a kernel gave up a bounded wait since the last call
 * (*detail, if non-null, receives the kernel-specific code), FA4Q_OK otherwise.
 */
fa4q_status fa4q_device_status(void* stream, uint32_t* detail);

/*
 * fa4q_selftest_wait_timeout - diagnostic: launch one kernel that waits, with the same
 * bounded-wait helper every pipelined kernel uses, on a barrier nothing will complete, for
 * `wait_us` microseconds.  The wait expires, the kernel records FA4Q_ERR_TIMEOUT in the
 * device status word and returns; no GPU hang or fault is involved.  Read it with
 * fa4q_device_status.  (Every pipelined kernel's waits give up after 2 s the same way.)
 */
fa4q_status fa4q_selftest_wait_timeout(uint32_t wait_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA4Q_H_ */
