/*
 * sage.h -- C ABI of libsage, a B200 (sm_100a) implementation of
 * SageAttention-style quantized attention with K smoothing.
 *
 * The path, in call order:
 *   sage_hadamard_init   once per head dimension: the rotation is fixed once
 *                        and reused for every call ("Sage v2 improvements":
 *                        the Hadamard matrix is created once and reused).
 *   sage_quant_qk        K smoothing (subtract K's per-(b,h) mean over the
 *                        sequence), Hadamard rotation of Q and K along the
 *                        head dim, INT8 quantisation with one absmax scale
 *                        per token block ("perf(dsv4): qproj wq_b transpose +
 *                        serving contract; ...", sequence diagram: Hadamard
 *                        transform -> per-head amax -> dequant scale -> INT8
 *                        rows).
 *   sage_quant_v         FP8 e4m3 quantisation of V with one scale per
 *                        channel ("Sage2 SM89 Temporal Pair Experiment",
 *                        Candidate: the kernel fuses a per-channel V scale).
 *   sage_quant_qkv       both of the above in one call (two launches: the K
 *                        and V statistics, then every Q, K and V tile), the
 *                        same outputs bit for bit.
 *   sage_attn_fwd        S = Q8 K8^T in INT8, dequantised, online softmax in
 *                        128-key tiles with the per-tile order QK ->
 *                        update_mdo -> accumulate_d -> RS_32_to_8 -> PV
 *                        ("Sage2 SM89 Temporal Pair Experiment", Candidate),
 *                        P cast to e4m3 after scaling by FP8_MAX = 448, PV in
 *                        FP8, epilogue x 1/FP8_MAX ("[FlyDSL] [Misc] pa_decode:
 *                        key the tile kernel on FlyDSL dtypes and drop the
 *                        batch-first plan grid", Changes), bf16 output.
 *   sage_attn_decode     paged FP8-KV decode (same page: window-family
 *                        workload, per-token FP8 K/V scales, MTP, GQA).
 *   sage_attn_decode_mxfp4  the same decode over an MXFP4 KV cache.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers on the device that is current
 *     for the calling thread, owned by the caller; the library never
 *     allocates, frees or copies them, never synchronises the stream (except
 *     sage_device_error) and never makes a contiguous copy ("Sage v2
 *     improvements": the forced .contiguous() was the bottleneck; "sage_attn3"
 *     API page: preprocess_qkv / postprocess_output permute-and-copy).
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream. Work is enqueued on it and the call returns at once.
 *   - Views (sage_cview4 / sage_view4) describe logical [B, H, L, D] tensors
 *     with sizes and strides counted in ELEMENTS (bf16), any non-negative
 *     strides; layouts that allow 16-byte vector access (unit D stride,
 *     other strides multiples of 8, 16-byte-aligned base) take the vector
 *     path, any other layout takes the scalar path with identical results.
 *   - Validation happens on the host before anything is launched; on error
 *     nothing is enqueued. Bad pointers/sizes/strides -> SAGE_ERR_INVALID_ARG,
 *     valid but unsupported shapes or formats -> SAGE_ERR_UNSUPPORTED (the
 *     FlyDSL page refuses unsupported dtypes the same two ways), a workspace
 *     that is too small -> SAGE_ERR_WORKSPACE, a failed CUDA launch ->
 *     SAGE_ERR_CUDA. Nothing aborts or traps.
 *   - Inputs must be finite; NaN/Inf inputs are outside the contract.
 *   - Every device wait inside the kernels is bounded; a wait that expires
 *     records an error word that sage_device_error reports as
 *     SAGE_ERR_TIMEOUT.
 *
 * Quantised buffer layouts (part of the contract; produced by the quant
 * entry points, consumed by sage_attn_fwd). Lpad(L) = L rounded up to 128.
 *   q8      int8   [B, H,  Lpad(Lq), D]  contiguous, rows >= Lq zero
 *   q_scale fp32   [B, H,  ceil(Lq / blk_q)]
 *   k8      int8   [B, Hk, Lpad(Lk), D]  contiguous, rows >= Lk zero
 *   k_scale fp32   [B, Hk, ceil(Lk / blk_k)]
 *   k_mean  fp32   [B, Hk, D]
 *   v8_t    e4m3   [B, Hk, D, Lpad(Lk)]  contiguous (V transposed: keys are
 *                                       the contiguous dim), columns >= Lk 0
 *   v_scale fp32   [B, Hk, D]
 */
#ifndef SAGE_H_
#define SAGE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sage_status {
    SAGE_OK = 0,
    SAGE_ERR_INVALID_ARG = 1,  /* null pointer, negative size/stride, bad handle */
    SAGE_ERR_UNSUPPORTED = 2,  /* valid but not supported (D, block size, page size, ...) */
    SAGE_ERR_ALIGNMENT = 3,    /* a quantised buffer is not 16-byte aligned */
    SAGE_ERR_WORKSPACE = 4,    /* workspace missing or smaller than *_workspace() */
    SAGE_ERR_CUDA = 5,         /* a CUDA runtime/driver call failed */
    SAGE_ERR_TIMEOUT = 6       /* a bounded device wait expired (see sage_device_error) */
} sage_status;

/* Read-only logical [B, H, L, D] view; sizes and strides in elements. */
typedef struct sage_cview4 {
    const void* ptr;
    int64_t size[4];
    int64_t stride[4];
} sage_cview4;

/* Writable logical [B, H, L, D] view; sizes and strides in elements. */
typedef struct sage_view4 {
    void* ptr;
    int64_t size[4];
    int64_t stride[4];
} sage_view4;

/* Opaque, immutable after init; usable from any stream and thread. */
typedef struct sage_hadamard_s* sage_hadamard;

/* Build the Sylvester Hadamard rotation H_D (entries +-1, H H^T = D I) for
 * head_dim D in {64, 128} once, for use with `device` ("Sage v2
 * improvements": created once, reused by every call). The kernels apply it
 * as the fp32 butterfly x -> x H (stages h = 1, 2, ..., D/2, each output one
 * IEEE add or subtract), unnormalised; the 1/D that Q H (K H)^T carries is
 * folded into the logit scale by sage_attn_fwd. The butterfly's pattern is
 * H, so the handle holds the matrix on the host only (sage_hadamard_matrix)
 * and no device memory. *out receives the handle.
 * Errors: INVALID_ARG (out NULL, device < 0 or past the device count),
 * UNSUPPORTED (other D), CUDA (device count unavailable). */
sage_status sage_hadamard_init(int head_dim, int device, sage_hadamard* out);

/* Free a handle from sage_hadamard_init (NULL is accepted). */
sage_status sage_hadamard_destroy(sage_hadamard h);

/* Copy H (row-major D x D, int8 +-1) to host memory `host_out` (D*D bytes)
 * and/or report D through `head_dim` (either may be NULL). */
sage_status sage_hadamard_matrix(sage_hadamard h, int8_t* host_out, int* head_dim);

/* Bytes of device workspace sage_quant_qk needs: the fp32 K mean of every
 * (b, kv head, d), passed from the statistics pass to the quantisation
 * pass: B * Hk * D * 4. */
size_t sage_quant_qk_workspace(int B, int H, int Hk, int Lq, int Lk, int D);

/* Smooth, rotate and INT8-quantise Q and K.
 *   q_bf16: [B, H, Lq, D] bf16 view;  k_bf16: [B, Hk, Lk, D] bf16 view;
 *   H % Hk == 0, D == handle's D, blk_q, blk_k in {32, 64, 128}.
 * Computes, per (b, h):
 *   mean_K[d] = fp32( (fp64 sum over the Lk tokens of K) / Lk )
 *   K_s = K - mean_K (fp32); Q is not smoothed;
 *   x_hat = butterfly(x) for every row of Q and K_s (fp32);
 *   per block of blk tokens: a = max|x_hat|, scale = a / 127,
 *   code = clamp(round_half_even(x_hat * (127 / a)), -127, 127) (a = 0 gives
 *   scale 0 and zero codes).
 * Writes q8, q_scale, k8, k_scale in the layouts above and, if k_mean is not
 * NULL, mean_K [B, Hk, D]. ws: device workspace of at least
 * sage_quant_qk_workspace(...) bytes, 16-byte aligned; its contents on
 * entry do not matter. Quantised outputs must be 16-byte aligned.
 * Results are bit-identical for any input strides. */
sage_status sage_quant_qk(sage_hadamard h, sage_cview4 q_bf16, sage_cview4 k_bf16, int blk_q,
                          int blk_k, int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                          float* k_mean, void* ws, size_t ws_bytes, void* stream);

/* The same computation and outputs as sage_quant_qk, for callers that cannot
 * allocate device memory when they quantise (for example a serving loop whose
 * device memory is budgeted once at start-up, or code that must not risk the
 * implicit device synchronisation cudaMalloc / cudaFree can cause). The
 * paper has no counterpart to this entry point; it is a property of this
 * library.
 * The scratch that sage_quant_qk takes as `ws` comes instead from a fixed
 * 8 MiB array built into the library; every GPU that loads the library holds
 * it until the process exits. Calls whose sage_quant_qk_workspace(...) exceeds
 * 8 MiB are rejected with SAGE_ERR_WORKSPACE before anything is launched
 * (8 MiB covers B * Hk * D <= 2 Mi, e.g. 16384 kv heads of D = 128).
 * The first call on a device looks the array's device address up
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture. Every call on a device shares the one array and leaves
 * its last contents there (each call writes every scratch entry it reads, so no
 * clearing is needed): calls that may run concurrently on the GPU (different
 * streams without ordering between them) race on it and must be serialised by
 * the caller. Allocates nothing; errors as for sage_quant_qk. */
sage_status sage_quant_qk_noalloc(sage_hadamard h, sage_cview4 q_bf16, sage_cview4 k_bf16,
                                  int blk_q, int blk_k, int8_t* q8, float* q_scale, int8_t* k8,
                                  float* k_scale, float* k_mean, void* stream);

/* sage_quant_qk for K alone (K mean, smoothing, rotation, INT8 codes and
 * scales, the same bits as sage_quant_qk's K outputs), for callers whose Q is
 * quantised inside sage_attn_fwd_q16. k_bf16: [B, Hk, Lk, D]; ws: at least
 * sage_quant_qk_workspace(B, Hk, Hk, Lk, Lk, D) bytes. */
sage_status sage_quant_k(sage_hadamard h, sage_cview4 k_bf16, int blk_k, int8_t* k8,
                         float* k_scale, float* k_mean, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace sage_quant_v needs: the fp32 multiplier 448 / a
 * of every (b, h, d): B * Hk * D * 4. */
size_t sage_quant_v_workspace(int B, int Hk, int L, int D);

/* FP8 e4m3 (OCP e4m3fn, max 448) per-channel quantisation of V.
 *   v_bf16: [B, Hk, L, D] bf16 view, D in {64, 128}.
 * Per (b, h, d): a = max over the L tokens of |v|, scale = a / 448,
 * code = e4m3_round_nearest_even_saturating(v * (448 / a)) (a = 0 gives
 * scale 0 and zero codes). Writes v8_t [B, Hk, D, Lpad(L)] (transposed) and
 * v_scale [B, Hk, D]. ws: at least sage_quant_v_workspace(...) bytes,
 * 16-byte aligned, contents on entry irrelevant. */
sage_status sage_quant_v(sage_cview4 v_bf16, uint8_t* v8_t, float* v_scale, void* ws,
                         size_t ws_bytes, void* stream);

/* Bytes of device workspace sage_quant_qkv needs:
 * sage_quant_qk_workspace(...) + sage_quant_v_workspace(B, Hk, Lk, D). */
size_t sage_quant_qkv_workspace(int B, int H, int Hk, int Lq, int Lk, int D);

/* sage_quant_qk and sage_quant_v in one call, with the same outputs bit for
 * bit: v_bf16 has k_bf16's sizes [B, Hk, Lk, D] (any strides). The K and V
 * statistics run as one launch and the Q, K and V quantisation as a second,
 * so the copy-bound V work shares the SMs with the Q/K rotation. ws: at
 * least sage_quant_qkv_workspace(...) bytes, 16-byte aligned, contents on
 * entry irrelevant. Errors as for sage_quant_qk, and INVALID_ARG when V's
 * sizes differ from K's. */
sage_status sage_quant_qkv(sage_hadamard h, sage_cview4 q_bf16, sage_cview4 k_bf16,
                           sage_cview4 v_bf16, int blk_q, int blk_k, int8_t* q8, float* q_scale,
                           int8_t* k8, float* k_scale, float* k_mean, uint8_t* v8_t,
                           float* v_scale, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace sage_attn_fwd needs (0 in this version). */
size_t sage_attn_fwd_workspace(int B, int H, int Hk, int Lq, int Lk, int D);

/* Quantised attention forward on the buffers written by the quant calls.
 * For query row i of head h (kv head h / (H / Hk)) and key j, with
 * c = softmax_scale / D:
 *   x_ij = (sum_d q8[i,d] k8[j,d]) * q_scale[i / blk_q] * k_scale[j / blk_k] * c
 *   causal != 0 masks j > i + (Lk - Lq) (bottom-right aligned).
 * Keys are processed in tiles of 128 in ascending order; per tile the
 * running max m and denominator d of each row are updated, P8 =
 * e4m3(448 * exp(x - m)) feeds an FP8 PV product, d sums the unquantised
 * probabilities, and out = bf16(O * v_scale / (448 * d)); a row that sees no
 * key is written as zeros. out_bf16: [B, H, Lq, D] bf16 view of any strides.
 * Supported: D in {64, 128}, blk_q and blk_k in {32, 64, 128}, Lq, Lk >= 1.
 * Pointers q8, k8, v8_t must be 16-byte aligned. ws may be NULL. */
sage_status sage_attn_fwd(const int8_t* q8, const float* q_scale, const int8_t* k8,
                          const float* k_scale, const uint8_t* v8_t, const float* v_scale, int B,
                          int H, int Hk, int Lq, int Lk, int D, int blk_q, int blk_k,
                          float softmax_scale, int causal, sage_view4 out_bf16, void* ws,
                          size_t ws_bytes, void* stream);

/* Q rotated and quantised inside the attention kernel: the per-token
 * rotate + absmax + INT8 step of the pypto DSV4 page ("qr_hadamard_quant")
 * fused into the attention CTA, on-chip, so the Q operand never round-trips
 * through HBM (that page fused it through global memory and lost). Each query row is read once as bf16, rotated with the butterfly and
 * quantised to INT8 with the block scale a / 127 of its blk_q-row block --
 * the arithmetic of sage_quant_qk, so the codes, scales and output are the
 * bits that sage_quant_qk + sage_attn_fwd produce -- and its codes go straight
 * into the shared-memory operand of QK. q8 / q_scale are never written.
 *   q_bf16: [B, H, Lq, D] bf16 view of any strides (D == the handle's D);
 *   k8, k_scale: from sage_quant_k (or sage_quant_qk) with the same blk_k;
 *   v8_t, v_scale: from sage_quant_v; out_bf16: [B, H, Lq, D] bf16 view.
 * Supported as for sage_attn_fwd. ws may be NULL. */
sage_status sage_attn_fwd_q16(sage_hadamard h, sage_cview4 q_bf16, int blk_q, const int8_t* k8,
                              const float* k_scale, const uint8_t* v8_t, const float* v_scale,
                              int Hk, int Lk, int blk_k, float softmax_scale, int causal,
                              sage_view4 out_bf16, void* ws, size_t ws_bytes, void* stream);

/* MXFP4 variant: Q and K quantised to OCP MX FP4 ("Sage v2 improvements",
 * Changelog: the fav3_sage_mxfp4 attention with a Hadamard block BLOCK_R =
 * 128, i.e. the whole head for D <= 128; "[FlyDSL] [Misc] pa_decode ...",
 * Changes: MXFP4 is packed E2M1 with float8_e8m0fnu scales, and Q / P use
 * E4M3 as their FP8 format). K is smoothed (its per-(b,h) mean subtracted,
 * as in sage_quant_qk) and Q and K rotated by the butterfly, then per row and
 * block of 32 consecutive elements: a = max |x_hat|, E = floor(log2 a) - 2
 * clamped to [-127, 125] (E = -127 for a = 0 or a subnormal a), codes
 * E2M1(x_hat * 2^-E) rounded to nearest even and saturating at 6 (a zero
 * block gets +0 codes), scale byte E + 127 (e8m0).
 *   q_bf16: [B, H, Lq, D], k_bf16: [B, Hk, Lk, D] bf16 views, D in {64, 128}
 *   (the handle's D), H % Hk == 0.
 * Layouts (16-byte aligned):
 *   q4 / k4    uint8 [B, H(k), Lpad, D/2]: element 2i of a row in the low
 *              nibble of byte i; rows >= L zero
 *   q_sf / k_sf uint8 [B, H(k), Lpad/128, 512]: per 128-row tile, the scale
 *              of row r, block j at byte 16 (r mod 32) + 4 (r div 32) + j
 *              (the order the block-scaled MMA reads); unused bytes zero
 * k_mean (nullable) and ws as for sage_quant_qk (ws: at least
 * sage_quant_qk_workspace(...) bytes). Errors as for sage_quant_qk. */
sage_status sage_quant_qk_mx(sage_hadamard h, sage_cview4 q_bf16, sage_cview4 k_bf16, uint8_t* q4,
                             uint8_t* q_sf, uint8_t* k4, uint8_t* k_sf, float* k_mean, void* ws,
                             size_t ws_bytes, void* stream);

/* Quantised attention with MXFP4 Q and K (from sage_quant_qk_mx) and FP8 V
 * (from sage_quant_v): for query row i of head h (kv head h / (H / Hk)) and
 * key j, with c = softmax_scale / D,
 *   x_ij = c * sum over 32-element blocks b of 2^(Eq_ib + Ek_jb) *
 *          sum_{d in b} e2m1(q_id) e2m1(k_jd)
 * (the block-scaled E2M1 MMA); then the per-tile sequence of sage_attn_fwd:
 * 128-key tiles, running max and denominator, P8 = e4m3(448 exp(x - m)), FP8
 * PV, out = bf16(O * v_scale / (448 d)); causal as for sage_attn_fwd.
 * out_bf16: [B, H, Lq, D] bf16 view of any strides. Supported: D in {64, 128},
 * softmax_scale > 0. ws may be NULL. */
sage_status sage_attn_fwd_mx(const uint8_t* q4, const uint8_t* q_sf, const uint8_t* k4,
                             const uint8_t* k_sf, const uint8_t* v8_t, const float* v_scale, int B,
                             int H, int Hk, int Lq, int Lk, int D, float softmax_scale, int causal,
                             sage_view4 out_bf16, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace sage_attn_decode needs on the current device:
 * the split-KV partials when the keys of a (sequence, kv head) are shared
 * out among several CTAs (at most one CTA per SM in all), 0 when B * Hk
 * reaches the SM count. No initial contents are required; concurrent calls
 * need distinct workspaces. */
size_t sage_attn_decode_workspace(int B, int T, int H, int Hk, int D, int window);

/* Cache variants of sage_attn_decode ("[FlyDSL] [Misc] pa_decode ...",
 * Performance: FP8 KV with per-tensor and per-token scales; Window-family
 * results: transposed V), OR-ed into kv_flags. */
#define SAGE_KV_PER_TENSOR_SCALES 1   /* k_scale / v_scale point to one fp32 each */
#define SAGE_KV_V_TRANSPOSED 2        /* v_cache is [num_pages, Hk, D, page], page 128 */

/* Paged FP8-KV decode with MTP query tokens and a sliding window.
 *   q_bf16: [B, T, H, D] bf16 view (the T query tokens are the last T
 *   positions of each sequence); k_cache, v_cache: e4m3 codes
 *   [num_pages, Hk, page_size, D] contiguous (v_cache [num_pages, Hk, D,
 *   page_size] with SAGE_KV_V_TRANSPOSED); k_scale, v_scale: fp32 per token
 *   [num_pages, Hk, page_size] (one fp32 each with SAGE_KV_PER_TENSOR_SCALES);
 *   page_table: int32 [B, max_pages]
 *   logical -> physical page; ctx_lens: int32 [B], T <= ctx <= max_pages *
 *   page_size. The cache holds keys already in the rotated domain. The
 *   kernel reads whole 128-key tiles and gives the keys outside a window a
 *   weight of exactly zero, multiplied by their v_scale: the per-token
 *   v_scale of every slot of the pages a window touches, and of page 0
 *   (it stands in for the pages of a tile that hold no window key), must be
 *   finite; codes and k_scale there may hold any bytes.
 * For token t (position p = ctx - T + t) and head h: q_hat = butterfly(q)
 * (fp32), per-(t, h) e4m3 quantisation with scale max|q_hat| / 448; keys j in
 * [max(0, p - window + 1), p]; S_j = (q8 . k8_j) * s_q * k_scale_j *
 * softmax_scale / D; softmax; out = sum_j p_j v_scale_j v8_j -> bf16.
 * out_bf16: [B, T, H, D] bf16 view. q8_out (nullable, 16-byte aligned):
 * receives the e4m3 codes of the rotated queries, contiguous [B, T, H, D];
 * q_scale_out (nullable): their scales s_q, contiguous fp32 [B, T, H] (the
 * codes the QK product used, for callers that reuse them or check them).
 * Supported: D in {64, 128} (D = 256 is UNSUPPORTED: its K/V stages, bf16
 * V and two O accumulators exceed one CTA's shared and tensor memory in
 * this pipeline), page_size in {16, 32, 64, 128}, H % Hk == 0,
 * H / Hk <= 16, T * (H / Hk) <= 64, window >= 1; SAGE_KV_V_TRANSPOSED
 * needs page_size 128 (UNSUPPORTED otherwise), unknown kv_flags bits are
 * INVALID_ARG. ws: at least sage_attn_decode_workspace(...) bytes, 16-byte
 * aligned. One kernel launch, or two when the keys of a (sequence, kv head)
 * are split among CTAs: the split kernel leaves (m, l, O) per CTA in ws and
 * a merge kernel combines them (log-sum-exp). */
sage_status sage_attn_decode(sage_hadamard h, sage_cview4 q_bf16, const uint8_t* k_cache,
                             const uint8_t* v_cache, const float* k_scale, const float* v_scale,
                             const int32_t* page_table, const int32_t* ctx_lens, int B, int T,
                             int H, int Hk, int D, int page_size, int max_pages, int num_pages,
                             int window, float softmax_scale, int kv_flags, sage_view4 out_bf16,
                             uint8_t* q8_out, float* q_scale_out, void* ws, size_t ws_bytes,
                             void* stream);

/* Paged decode over an MXFP4 cache ("[FlyDSL] [Misc] pa_decode ...",
 * Changes: a uint8 cache is MXFP4, packed E2M1 with e8m0 scales, and the
 * query is quantised to E4M3 for it; Performance: MXFP4 KV, GQA 16, page
 * 128, batch 1 / 32 / 256, ctx 2k / 32k).
 *   k_cache, v_cache: E2M1 codes [num_pages, Hk, page_size, D / 2] bytes,
 *   contiguous, element 2i in the low nibble of byte i and 2i + 1 in the
 *   high one (nibble: sign, two exponent bits, one mantissa bit: 0, 0.5, 1,
 *   1.5, 2, 3, 4, 6); k_sf, v_sf: e8m0 block scales [num_pages, Hk,
 *   page_size, D / 32] bytes, contiguous, 16-byte aligned: element e of a
 *   token is code(e) * 2^(sf[e / 32] - 127). Everything else is as for
 *   sage_attn_decode (same query quantisation, windows, q8_out /
 *   q_scale_out, workspace and launches) with k_scale = v_scale = 1: S_j =
 *   (q8 . k_j) * s_q * softmax_scale / D; out = sum_j p_j v_j -> bf16, the
 *   weights p_j rounded to bf16 before the PV product. The dequantised K and
 *   V are exact in bf16 for scale codes 0 .. 252; codes 253 .. 255
 *   (values beyond the bf16 range, and NaN) are outside the contract and
 *   read as 252, so the unused slots of the pages a window touches may hold
 *   any bytes. Supported: D = 128 (other D: UNSUPPORTED), page_size in
 *   {16, 32, 64, 128}, H % Hk == 0, H / Hk <= 16, T * (H / Hk) <= 64. */
sage_status sage_attn_decode_mxfp4(sage_hadamard h, sage_cview4 q_bf16, const uint8_t* k_cache,
                                   const uint8_t* v_cache, const uint8_t* k_sf, const uint8_t* v_sf,
                                   const int32_t* page_table, const int32_t* ctx_lens, int B, int T,
                                   int H, int Hk, int D, int page_size, int max_pages, int num_pages,
                                   int window, float softmax_scale, sage_view4 out_bf16,
                                   uint8_t* q8_out, float* q_scale_out, void* ws, size_t ws_bytes,
                                   void* stream);

/* Static, human-readable name of a status code. */
const char* sage_status_string(sage_status s);

/* Synchronise `stream`, then read and clear the library's device error
 * words on the current device: SAGE_ERR_TIMEOUT if a bounded wait expired
 * since the last call, SAGE_ERR_CUDA if the stream reports a CUDA error,
 * SAGE_ERR_INVALID_ARG if sage_attn_decode met device-side arguments out of
 * range (a context length above max_pages * page_size, clamped; or a page id
 * outside [0, num_pages) for a page holding keys of a window, whose keys were
 * then left out), SAGE_OK otherwise. */
sage_status sage_device_error(void* stream);

/* Kernel ids reported by sage_device_error_where. */
#define SAGE_KERNEL_ATTN 1
#define SAGE_KERNEL_DECODE 2
#define SAGE_KERNEL_PROBE 3
#define SAGE_KERNEL_ATTN_MX 4

/* sage_device_error, also saying where the reported error was recorded:
 * *kernel receives a SAGE_KERNEL_* id (0 with SAGE_OK), *site the number of
 * the wait (or check) inside that kernel that recorded it. Either pointer
 * may be NULL. Reads and clears the same error words as sage_device_error. */
sage_status sage_device_error_where(void* stream, int* kernel, int* site);

/* Failure-path probe (diagnostic; no page counterpart): enqueue one small
 * kernel whose bounded mbarrier wait is never satisfied. The wait gives up
 * after limit_ns nanoseconds (1 us .. 10 s), records a timeout at site 1 of
 * SAGE_KERNEL_PROBE and raises its CTA's abort flag; a second waiter of the
 * CTA (the kernels' default 2 s limit) must then end early through that
 * flag, and the TMEM the CTA holds is released -- the path every kernel of
 * the library takes when one of its waits expires. The next
 * sage_device_error_where on `stream` reports SAGE_ERR_TIMEOUT, kernel 3,
 * site 1; the device stays usable. Errors: INVALID_ARG (limit out of range),
 * CUDA (launch failed). */
sage_status sage_wait_probe(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_H_ */
