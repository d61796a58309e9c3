/*
 * moe.h -- C ABI of libmoe, the routed 4-bit mixture-of-experts FFN for B200
 * (sm_100a).
 *
 * The operation: a token's router logits pick k of E experts by softmax and
 * renormalised top-k; each picked expert applies a SwiGLU FFN
 * (gate/up: H -> F, SiLU(gate) * up, down: F -> H) whose weights are stored as
 * 4-bit codes; the k expert outputs are summed with the routing weights.
 * Sources, by page title and section:
 *   - "Drama 3 int4 (drama-rs format)", section "What's quantized": routed
 *     experts are int4, asymmetric, group 64, f16 scale + min.
 *   - "drama-rs", section "Apple Silicon (MLX)": the same values map to the
 *     packed affine form w = q * scale + min; prefill groups rows by routed
 *     expert; section "Footprint and speed": decode is weight streaming.
 *   - "Drama 3 - NVFP4 routed experts", section "Quantization": 40 layers x 256
 *     experts x 3 projections; the NVFP4 variant (E2M1 codes, E4M3 scale per 16
 *     input channels, FP32 global scale per matrix shared by gate and up,
 *     dynamic per-token activation scales).
 *
 * Conventions (every call):
 *   - Returns moe_status; argument errors are found on the host before any
 *     launch and nothing is enqueued then.  MOE_ERR_CUDA reports a launch
 *     error (the CUDA error string is kept for moe_last_error_string()).
 *   - Every array argument is a DEVICE pointer owned by the caller, unless the
 *     comment says "host".  The library allocates no memory: calls that need
 *     scratch take a caller workspace sized by the matching *_workspace_bytes()
 *     query.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; nothing synchronises.
 *   - bf16 and f16 values travel as uint16_t bit patterns.
 *   - Inputs must be finite; NaN logits or activations give unspecified
 *     (but memory-safe) results.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_API __attribute__((visibility("default")))

typedef void *moe_stream_t; /* a cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,       /* null pointer, negative size, k > E, ... */
  MOE_ERR_UNSUPPORTED_SHAPE = 2, /* a size this library's kernels do not tile */
  MOE_ERR_WORKSPACE = 3,         /* workspace missing or smaller than required */
  MOE_ERR_CUDA = 4,              /* a CUDA launch or runtime call failed */
  MOE_ERR_TIMEOUT = 5            /* a bounded device-side wait gave up */
} moe_status;

/* Human-readable name of a status code (static string). */
MOE_API const char *moe_status_string(moe_status s);
/* Text of the last CUDA error seen by this thread (static storage). */
MOE_API const char *moe_last_error_string(void);
/* Library version string, e.g. "moe-w4-b200 1". */
MOE_API const char *moe_version(void);

/* ======================================================================== */
/* int4 expert weights                                                       */
/* ======================================================================== */
/*
 * Canonical form of one [N][K] matrix (K = input channels):
 *   codes u8 [N][K], values 0..15
 *   scale f16 [N][K/64], min f16 [N][K/64]: group g of row n covers
 *   channels [64g, 64g + 64); the weight is codes * scale + min.
 * A gate/up pair is one canonical [2F][H] matrix: rows [0, F) gate, rows
 * [F, 2F) up.
 *
 * Device ("packed") form, written by moe_pack_w4 and read by every kernel:
 * 16-row strips, each strip a run of K/64 blocks of 576 bytes (512 bytes of
 * codes in the register order of the decode kernel's tensor-core fragments,
 * then 16 x {f16 scale, f16 min}).  Size: moe_w4_packed_bytes(N, K) =
 * N * K * 9 / 16 bytes.  For kind MOE_W4_GATE_UP the gate strip i and the up
 * strip i (same 16 features) are stored next to each other.
 * Requirements: N % 16 == 0 (gate/up: F % 16 == 0), K % 64 == 0.
 */
typedef enum { MOE_W4_PLAIN = 0, MOE_W4_GATE_UP = 1 } moe_w4_kind;

MOE_API size_t moe_w4_packed_bytes(int N, int K);

/*
 * Quantise fp32 weights w [N][K] to the canonical int4 form (group 64 along K,
 * asymmetric): per group m = f16(min) rounded toward -inf, s = f16((max - m)/15)
 * rounded toward +inf, q = clamp(rint((w - m) / s), 0, 15) in fp32 (s = 0 gives
 * q = 0).  Outputs codes [N][K], scale [N][K/64], min [N][K/64].
 * Source: "Drama 3 int4 (drama-rs format)", "What's quantized" (asymmetric,
 * group 64, f16 scale + min); plain min/max instead of the page's MSE clip
 * search.  Errors: INVALID_ARG (null, N or K < 0), UNSUPPORTED_SHAPE (K % 64).
 */
MOE_API moe_status moe_quantize_w4(const float *w, int N, int K, uint8_t *codes,
                                   uint16_t *scale, uint16_t *minv, moe_stream_t stream);

/*
 * The same format with the MSE clip search: for every group, 20 candidate
 * ranges, the group's [min, max] scaled by p_i = (100 - i) / 100 (i = 0..19,
 * 1.0 down to 0.81), each rounded as above (m toward -inf, s toward +inf from
 * the rounded m) and coded by nearest rounding; the candidate with the
 * smallest fp32 sum over the group, in channel order, of (q*s + m - w)^2 wins,
 * ties to the larger ratio.  p = 1 is exactly moe_quantize_w4's choice, so
 * no group gets a larger squared error.  Every step is one correctly rounded
 * fp32 operation, so the choice and the codes do not depend on the device.
 * Source: "Drama 3 int4 (drama-rs format)", table "What's quantized" (MSE
 * clip search); "drama-3-w4a16", section "How it was made" (20 clipping
 * ratios 1.0 -> 0.81 by minimum squared error).  Errors as moe_quantize_w4.
 */
MOE_API moe_status moe_quantize_w4_clip(const float *w, int N, int K, uint8_t *codes,
                                        uint16_t *scale, uint16_t *minv, moe_stream_t stream);

/*
 * Symmetric group-128 int4 ("drama-3-w4a16", table "At a glance": int4,
 * symmetric, group 128, GPTQ packing; section "How it was made": one scale
 * per 128 input weights, round-to-nearest, clip search as above):
 *   w = (q - 8) * s,  q in 0..15 (GPTQ's zero point 8), s f16 per 128 inputs,
 *   candidate s_i = f16(2 * (p_i * amax) / 15) nearest-even,
 *   q = clamp(rint(w / s) + 8, 0, 15) (s == 0 gives q = 8).
 * Outputs codes u8 [N][K] and scale f16 [N][K/128].  Errors: INVALID_ARG,
 * UNSUPPORTED_SHAPE (K % 128).
 */
MOE_API moe_status moe_quantize_w4_sym128(const float *w, int N, int K, uint8_t *codes,
                                          uint16_t *scale, moe_stream_t stream);

/*
 * Packs a symmetric group-128 matrix (codes [N][K], scale [N][K/128]) into the
 * int4 device form above, so every int4 kernel runs it unchanged: each group
 * of 128 becomes two groups of 64 with scale s and min -8 s, and q*s + (-8 s)
 * equals (q - 8) * s exactly.  Requires |s| < 8192 (so that -8 s is an f16).
 * ws: moe_pack_w4_sym128_workspace_bytes(N, K) bytes of scratch, 4-byte
 * aligned.  Errors: as moe_pack_w4, UNSUPPORTED_SHAPE for K % 128, WORKSPACE.
 */
MOE_API size_t moe_pack_w4_sym128_workspace_bytes(int N, int K);
MOE_API moe_status moe_pack_w4_sym128(const uint8_t *codes, const uint16_t *scale, int N, int K,
                                      int kind, void *packed, size_t packed_bytes, void *ws,
                                      size_t ws_bytes, moe_stream_t stream);

/* Canonical -> packed.  packed_bytes must be >= moe_w4_packed_bytes(N, K).
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (N % 16, K % 64, GATE_UP with N % 32),
 * WORKSPACE (packed_bytes too small). */
MOE_API moe_status moe_pack_w4(const uint8_t *codes, const uint16_t *scale,
                               const uint16_t *minv, int N, int K, int kind, void *packed,
                               size_t packed_bytes, moe_stream_t stream);

/* Packed -> canonical (exact inverse of moe_pack_w4). */
MOE_API moe_status moe_unpack_w4(const void *packed, int N, int K, int kind, uint8_t *codes,
                                 uint16_t *scale, uint16_t *minv, moe_stream_t stream);

/* Packed -> dequantised fp32 [N][K] in canonical row order, each weight one
 * fp32 fused multiply-add q * s + m (the value the oracle's dequant gives,
 * bit for bit).  A test and debugging export; kernels never materialise it. */
MOE_API moe_status moe_dequant_w4(const void *packed, int N, int K, int kind, float *out,
                                  moe_stream_t stream);

/*
 * One MoE layer's experts, all in device memory, experts stored back to back:
 *   gate_up: E * moe_w4_packed_bytes(2F, H) bytes, expert e at
 *            e * moe_w4_packed_bytes(2F, H), packed with kind MOE_W4_GATE_UP
 *   down:    E * moe_w4_packed_bytes(H, F) bytes, kind MOE_W4_PLAIN
 * The struct itself is a HOST struct passed by pointer; it is read during
 * the call only.
 */
typedef struct {
  int E, H, F;
  const void *gate_up;
  const void *down;
} moe_w4_layer;

/* ======================================================================== */
/* NVFP4 expert weights and activations (the variant)                        */
/* ======================================================================== */
/*
 * Source: "Drama 3 - NVFP4 routed experts", section "Quantization": E2M1
 * codes, one E4M3 scale per 16 input channels, one FP32 global scale per
 * matrix with gate and up sharing theirs, round to nearest; activations are
 * quantised dynamically per token (FP32 global, E4M3 block scales).  The
 * formulas are this library's reading:
 *   G   = amax / 2688 (= 448 * 6), or 1 when amax == 0
 *   S_b = E4M3(amax_b / (6 G)), nearest-even, saturating at 448
 *   q_i = E2M1(v_i / (S_b G)), nearest-even, saturating at +-6; 0 if S_b == 0
 * each division and product one correctly rounded fp32 operation; the value
 * of q_i is E2M1(q_i) * S_b * G.
 * Canonical form of one [N][K] matrix: codes u8 [N][K] (E2M1 bit patterns
 * 0..15, bit 3 the sign), sf u8 [N][K/16] (E4M3 bit patterns), and G.
 * Device ("packed") form, moe_nvfp4_packed_bytes(N, K) = N * K * 9 / 16
 * bytes: 16-row strips (gate/up: gate strip i next to up strip i, as for
 * int4), each strip 16 rows of K/2 code bytes (logical byte b holds channel
 * 2b in its low nibble; inside each 128-byte run of row r the 16-byte pieces
 * are XOR-permuted by r & 7, the tensor cores' 128-byte shared-memory
 * swizzle) followed by the scales as [K/64][16 rows][4] bytes.
 * Requirements: N % 16 == 0 (gate/up: N % 32 == 0), K % 256 == 0.
 */
MOE_API size_t moe_nvfp4_packed_bytes(int N, int K);

/* Device scalar *G = the global scale of n fp32 values v (formula above).
 * G is also the scratch of the reduction; n == 0 gives 1.  Errors:
 * INVALID_ARG. */
MOE_API moe_status moe_nvfp4_global(const float *v, size_t n, float *G, moe_stream_t stream);

/* Quantise fp32 v [N][K] with the device global *G to the canonical form:
 * codes u8 [N][K], sf u8 [N][K/16].  v and codes 16-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (K % 16). */
MOE_API moe_status moe_quantize_nvfp4(const float *v, int N, int K, const float *G,
                                      uint8_t *codes, uint8_t *sf, moe_stream_t stream);

/* Canonical -> packed, and its exact inverse.  Errors as for moe_pack_w4
 * (UNSUPPORTED_SHAPE for K % 256). */
MOE_API moe_status moe_pack_nvfp4(const uint8_t *codes, const uint8_t *sf, int N, int K,
                                  int kind, void *packed, size_t packed_bytes,
                                  moe_stream_t stream);
MOE_API moe_status moe_unpack_nvfp4(const void *packed, int N, int K, int kind,
                                    uint8_t *codes, uint8_t *sf, moe_stream_t stream);

/*
 * Per-row (per-token) activation quantisation, one global per row:
 * output row p quantises input row src = src_rows ? src_rows[p] / src_div : p
 * of x ([*][K], bf16 when x_dtype == 0, fp32 when x_dtype == 1).  Outputs:
 * codes u8 [rows][K/2] (two per byte, channel 2b in the low nibble of byte b),
 * sf u8 [rows][K/16], G fp32 [rows].  With src_rows = sorted_rows and
 * src_div = k (from moe_permute) this quantises and groups the rows by
 * expert in one pass.  x 16-byte aligned, codes 8-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (K % 16).
 */
MOE_API moe_status moe_quantize_nvfp4_rows(const void *x, int x_dtype, int rows, int K,
                                           const int32_t *src_rows, int src_div,
                                           uint8_t *codes, uint8_t *sf, float *G,
                                           moe_stream_t stream);

/*
 * One MoE layer's NVFP4 experts, experts back to back as for moe_w4_layer
 * (gate_up: E * moe_nvfp4_packed_bytes(2F, H), kind MOE_W4_GATE_UP; down:
 * E * moe_nvfp4_packed_bytes(H, F), kind MOE_W4_PLAIN), with device arrays of
 * the experts' globals g_gu [E] (shared by gate and up) and g_d [E].  A HOST
 * struct read during the call only.
 */
typedef struct {
  int E, H, F;
  const void *gate_up;
  const void *down;
  const float *g_gu;
  const float *g_d;
} moe_nvfp4_layer;

/* ======================================================================== */
/* Routing and permutation                                                   */
/* ======================================================================== */

/*
 * Top-k routing of T tokens over E experts from fp32 logits [T][E].
 * idx [T][k]: the k largest logits' expert ids, larger logit first, equal
 * logits to the lower expert id first.  w [T][k]: softmax over all E,
 * restricted to the selected experts and renormalised to sum to one (equal to
 * the softmax of the selected logits).  Source: the router of "Drama 3 int4",
 * "What's quantized" (bf16 router); top-k, renormalisation and tie order are
 * this library's reading.  Limits: 1 <= k <= min(E, 32), E <= 1024.
 * T == 0 is a no-op.  Errors: INVALID_ARG, UNSUPPORTED_SHAPE.
 */
MOE_API moe_status moe_route(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                             moe_stream_t stream);

/*
 * moe_route with a shared expert: the same routing of logits [T][E] over the
 * E routed experts, written to rows of k + 1 entries, the last one the shared
 * expert (id E, weight 1).  idx, w [T][k+1].  With moe_permute over E + 1
 * experts and moe_unpermute_combine with k + 1 rows, the layer output is the
 * routed sum plus the shared expert's row, added last.
 * Source: a shared expert beside the routed ones ("Drama 3 int4 (drama-rs
 * format)", table "What's quantized"; "Drama 3 - NVFP4 routed experts",
 * "Quantization"); weight 1 and the order of the sum are this library's
 * reading.  Limits: 1 <= k <= min(E, 31), E <= 1023.  T == 0 is a no-op.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE.
 */
MOE_API moe_status moe_route_shared(const float *logits, int T, int E, int k, int32_t *idx,
                                    float *w, moe_stream_t stream);

/*
 * The router linear fused with routing: logits[t][e] = sum_k x[t][k] *
 * Wr[e][k] (x bf16 [T][H], Wr bf16 [E][H], fp32 products and sums, no bias),
 * then the routing of moe_route on those logits (idx, w as there).  Up to 16
 * tokens one launch does both (the last CTA to finish its logits routes);
 * above, a tensor-core GEMM launch is followed by moe_route's kernel, chained
 * by programmatic dependent launch.  logits fp32 [T][E] is an optional
 * output (NULL: kept in the workspace).  For a decode layer,
 * moe_decode_layer_w4a16_router computes the router inside the layer's own
 * launch instead.  Source: the router stays bf16 ("Drama 3 int4 (drama-rs
 * format)", table "What's quantized"; "DRAMA-3 MLX expert-only 4-bit",
 * section "Quantization and provenance"); fp32 accumulation and no bias are
 * this library's reading.  The products are summed in the kernel's own
 * fixed order (fp32 FMAs in a fixed tree up to 16 tokens, the tensor cores
 * above), so logits can differ from a sequential fp32 sum in the last bits
 * but not from call to call; the selection is made on the logits this call
 * computes.
 * Workspace: moe_router_route_workspace_bytes(T, E) bytes, 16-byte aligned,
 * zero-filled before its first use; every call leaves it ready for the next
 * stream-ordered call.  Limits: E % 16 == 0 (E % 64 == 0 above 64), E <=
 * 1024, H % 64 == 0, 1 <= k <= min(E, 32).  x, Wr 16-byte aligned, logits
 * 8-byte aligned.  T == 0 is a no-op.  Errors: INVALID_ARG,
 * UNSUPPORTED_SHAPE, WORKSPACE, CUDA.
 */
MOE_API size_t moe_router_route_workspace_bytes(int T, int E);
MOE_API moe_status moe_router_route(const uint16_t *x, const uint16_t *wr, int T, int E, int H, int k,
                                    float *logits, int32_t *idx, float *w, void *ws, size_t ws_bytes,
                                    moe_stream_t stream);

/*
 * Group the T*k rows r = t*k + j by expert idx[r] (stable: within an expert,
 * rows in increasing r).  Outputs counts [E], offsets [E+1] (exclusive scan,
 * offsets[E] = T*k), sorted_rows [T*k] (row ids in grouped order), inv [T*k]
 * (inv[r] = position of row r).  If x (bf16 [T][H]) and x_perm are non-null,
 * also gathers x_perm[p] = x[sorted_rows[p] / k] (bf16 [T*k][H], H % 8 == 0).
 * Source: "drama-rs", "Apple Silicon (MLX)": prefill groups rows by routed
 * expert.  Counting is deterministic and uses no global atomics.
 * Workspace: moe_permute_workspace_bytes(T, k, E).  idx values must lie in
 * [0, E).  Errors: INVALID_ARG, UNSUPPORTED_SHAPE, WORKSPACE.
 */
MOE_API size_t moe_permute_workspace_bytes(int T, int k, int E);
MOE_API moe_status moe_permute(const int32_t *idx, int T, int k, int E, const uint16_t *x,
                               int H, int32_t *counts, int32_t *offsets, int32_t *sorted_rows,
                               int32_t *inv, uint16_t *x_perm, void *ws, size_t ws_bytes,
                               moe_stream_t stream);

/* ======================================================================== */
/* Expert FFN                                                                */
/* ======================================================================== */

/*
 * Decode: the expert FFN of every row r = t*k + j, expert idx[r], on x[t]:
 *   g, u = W_gate x, W_up x;  h = SiLU(g) * u;  y_rows[r] = W_down h
 * for a small batch (1 <= T <= 16 tokens, T*k <= 256), streaming each selected
 * expert's int4 weights from HBM once per call whatever the number of tokens
 * routed to it.  x bf16 [T][H]; idx [T][k] (from moe_route); y_rows fp32
 * [T*k][H].  Accumulation is fp32; h is rounded to bf16 before the down
 * projection.  Source: "drama-rs", "Footprint and speed" (decode is weight
 * streaming GEMVs) and "Experts: where they run" (decode is memory-bandwidth
 * bound); the SwiGLU expert of the Qwen3.5-MoE backbone.
 * Workspace: moe_decode_workspace_bytes(T, k, F) bytes (a call counter and
 * the h handoff buffer), 16-byte aligned.  Zero-fill it once before its
 * first use; every call leaves it ready for the next stream-ordered call, so
 * one workspace serves any number of calls.  Calls that share a workspace
 * must not overlap in time.  After a call that raised the device error word,
 * zero-fill the workspace again.
 * Requirements: H % 64 == 0, F % 64 == 0, idx values in [0, E), the k
 * experts of a token distinct.  Errors: INVALID_ARG, UNSUPPORTED_SHAPE,
 * WORKSPACE, CUDA.  A device-side wait that times out (it cannot under the
 * requirements above) raises the device error word: see moe_device_error().
 * Co-residency: the kernel's thread blocks (one per SM, at most the SM count)
 * wait on one another's results, so all of them must run at the same time.
 * The launch is cooperative: while other work (another stream, another
 * process under MPS) holds SMs, the GPU starts the grid only once every block
 * can run, instead of starting part of it.  The same holds for
 * moe_decode_layer_w4a16, moe_decode_layer_w4a16_shared,
 * moe_decode_layer_w4a16_router, moe_decode_layer_nvfp4 and
 * moe_ffn_w4a16_decode_static.
 */
MOE_API size_t moe_decode_workspace_bytes(int T, int k, int F);
MOE_API moe_status moe_ffn_w4a16_decode(const moe_w4_layer *layer, const uint16_t *x,
                                        const int32_t *idx, int T, int k, float *y_rows,
                                        void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * One whole MoE layer for a small batch in a single launch: routing (as
 * moe_route, bit-identical), the weight-streaming expert FFN (as
 * moe_ffn_w4a16_decode) and the router-weighted combine (as
 * moe_unpermute_combine: j ascending, fp32, nearest-even bf16).
 *   x bf16 [T][H], logits fp32 [T][E] -> y bf16 [T][H];
 *   idx [T][k] / w [T][k]: optional outputs of the routing (both or neither).
 * Workspace: moe_decode_layer_workspace_bytes(T, k, H, F) bytes, 16-byte
 * aligned, zero-filled before first use, reusable by stream-ordered calls
 * (as for moe_ffn_w4a16_decode).  Limits: 1 <= T <= 16, T*k <= 256,
 * k <= 32, E <= 1024, H % 64 == 0, F % 64 == 0.  Each 64-output chunk of a
 * token is summed by the last of its k down-projection work items, in j
 * order, so the result does not depend on scheduling.
 * Source: the same passages as moe_route, moe_ffn_w4a16_decode and
 * moe_unpermute_combine ("Footprint and speed": a decode step is streamed
 * weight GEMVs, here one launch per layer).
 */
MOE_API size_t moe_decode_layer_workspace_bytes(int T, int k, int H, int F);
MOE_API moe_status moe_decode_layer_w4a16(const moe_w4_layer *layer, const uint16_t *x,
                                          const float *logits, int T, int k, uint16_t *y,
                                          int32_t *idx, float *w, void *ws, size_t ws_bytes,
                                          moe_stream_t stream);

/*
 * moe_decode_layer_w4a16 with a shared expert.  `layer` holds E = Er + 1
 * experts: the Er routed ones, then the shared expert (id Er).  logits fp32
 * [T][Er]; each token runs its k routed experts and the shared one, and
 *   y = bf16( (sum over j < k, ascending, of w[t][j] * row(t, j)) + row(t, shared) )
 * in fp32, as moe_route_shared + moe_unpermute_combine with k + 1 rows.
 * idx, w [T][k]: optional outputs of the routed selection (both or neither).
 * Workspace: moe_decode_layer_workspace_bytes(T, k + 1, H, F).  Limits as
 * for moe_decode_layer_w4a16 with k + 1 in place of k (T*(k+1) <= 256,
 * k + 1 <= 32, E <= 1024).  Source: the passages of moe_route_shared and
 * moe_decode_layer_w4a16.
 */
MOE_API moe_status moe_decode_layer_w4a16_shared(const moe_w4_layer *layer, const uint16_t *x,
                                                 const float *logits, int T, int k, uint16_t *y,
                                                 int32_t *idx, float *w, void *ws, size_t ws_bytes,
                                                 moe_stream_t stream);

/*
 * The decode layer with the router linear inside the same launch: the kernel
 * computes logits[t][e] = sum_c x[t][c] * Wr[e][c] (x and Wr bf16 [E - shared]
 * [H], fp32 FMAs, no bias) for the routed experts, routes on them as
 * moe_route, and runs the layer as moe_decode_layer_w4a16 (shared = 0) or
 * moe_decode_layer_w4a16_shared (shared = 1: the layer's last expert is the
 * shared expert).  Each expert row's logits are summed by one warp: lane l
 * takes channels 8l .. 8l+7 of every 256 in order, then the 32 lanes' sums
 * meet in a fixed xor-shuffle tree, so the logits do not change from call to
 * call; they can differ from moe_router_route's (another order) in the last
 * bits.  logits fp32 [T][E - shared], idx / w [T][k]: optional outputs
 * (idx and w both or neither).  Wr 16-byte aligned.
 * Workspace: moe_decode_layer_router_workspace_bytes(T, k, shared, E, H, F)
 * (E = layer->E), zero-filled before first use, reusable by stream-ordered
 * calls.  Limits as for the call it extends.  A wait for a logit that times
 * out (it cannot while every block is resident) raises
 * MOE_DEVERR_DECODE_ROUTER_WAIT.  Source: the router stays bf16 ("Drama 3
 * int4 (drama-rs format)", table "What's quantized"; "DRAMA-3 MLX
 * expert-only 4-bit", "Quantization and provenance"), and the passages of the
 * calls it extends.
 */
MOE_API size_t moe_decode_layer_router_workspace_bytes(int T, int k, int shared, int E, int H, int F);
MOE_API moe_status moe_decode_layer_w4a16_router(const moe_w4_layer *layer, const uint16_t *x,
                                                 const uint16_t *wr, int T, int k, int shared,
                                                 uint16_t *y, int32_t *idx, float *w, float *logits,
                                                 void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The NVFP4 form of moe_decode_layer_w4a16: one launch routes the T tokens,
 * quantises each token's x to NVFP4 (per-token global, as
 * moe_quantize_nvfp4_rows), runs every selected expert's FFN on the NVFP4
 * weights of `layer` (fp32 sums of E2M1 * E4M3 products per 16-channel block,
 * times the two globals; gate and up outputs scaled before SwiGLU), quantises
 * each row's fp32 h to NVFP4 (per-row global) before the down projection, and
 * writes the router-weighted combine y bf16 [T][H].
 * Source: "Drama 3 - NVFP4 routed experts", section "Quantization" (NVFP4
 * weights, dynamic per-token activation scales), and the passages of
 * moe_decode_layer_w4a16.
 * Workspace: moe_decode_layer_workspace_bytes(T, k, H, F), as for the int4
 * form.  Limits as for moe_decode_layer_w4a16, with H % 256 == 0 and
 * F % 256 == 0.
 */
MOE_API moe_status moe_decode_layer_nvfp4(const moe_nvfp4_layer *layer, const uint16_t *x,
                                          const float *logits, int T, int k, uint16_t *y,
                                          int32_t *idx, float *w, void *ws, size_t ws_bytes,
                                          moe_stream_t stream);

/*
 * Allocation-free form of moe_ffn_w4a16_decode (the pages have no counterpart;
 * this is a library convenience).  Same inputs, outputs and results, but no
 * workspace argument: the scratch lives in one fixed array of 516 KiB
 * (4 KiB of counter words + 512 KiB of h handoff words) inside the library's
 * device memory,
 * which every GPU that loads the library keeps until the process exits.  It
 * is for callers that cannot allocate device memory, such as plugins whose
 * host application owns and budgets all device memory, or programs with a
 * fixed memory plan that forbids allocation once serving has started.
 *   - Limit: T * k * F * 8 <= 512 KiB (one 8-byte handoff word per h value;
 *     e.g. T*k = 128 rows at F = 512);
 *     larger calls return MOE_ERR_WORKSPACE.  Other limits as for
 *     moe_ffn_w4a16_decode.
 *   - Allocates nothing: no cudaMalloc, no cudaFree.  Each call clears the
 *     CTA counter word with a cudaMemsetAsync on `stream`, then launches the
 *     kernel; the call-number word keeps counting across calls.
 *   - The first call on a device looks up the array's device address on that
 *     (current) device; make that first call before any stream capture.  The
 *     address is cached per device for the life of the process: after a
 *     cudaDeviceReset it is stale, so do not call this function again on
 *     that device.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind: two calls whose executions overlap on the GPU (different
 *     streams, no ordering between them) race and give wrong results.
 */
MOE_API moe_status moe_ffn_w4a16_decode_static(const moe_w4_layer *layer, const uint16_t *x,
                                               const int32_t *idx, int T, int k, float *y_rows,
                                               moe_stream_t stream);

/*
 * Prefill: grouped GEMM over experts.  x_perm bf16 [rows][H] holds the rows
 * grouped by expert (from moe_permute), offsets [E+1] (device) delimits the
 * groups.  Writes y_perm bf16 [rows][H] = W_down (SiLU(W_gate x) * W_up x)
 * for every row with its group's expert, on the tensor cores (tcgen05, fp32
 * accumulation in tensor memory, h rounded to bf16).
 * Source: "drama-rs", "Layout" (prefill: grouped MoE) and "Apple Silicon
 * (MLX)" (prefill groups rows by routed expert).
 * Workspace: moe_prefill_workspace_bytes(rows, F) bytes, 16-byte aligned.
 * After the call its first rows * F * 2 bytes hold h (bf16 [rows][F], the
 * gate/up stage, in the same grouped row order), for stage-wise checks.
 * Requirements: H % 256 == 0, F % 128 == 0, E <= 960,
 * offsets non-decreasing with offsets[0] == 0 and offsets[E] == rows.
 * rows == 0 is a no-op.
 */
MOE_API size_t moe_prefill_workspace_bytes(int rows, int F);
MOE_API moe_status moe_ffn_grouped_prefill(const moe_w4_layer *layer, const uint16_t *x_perm,
                                           const int32_t *offsets, int rows, uint16_t *y_perm,
                                           void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Prefill with NVFP4 experts: grouped GEMM over experts on the block-scaled
 * tensor cores (tcgen05 kind::mxf4nvf4: E2M1 x E2M1 with E4M3 scales per 16
 * channels, fp32 accumulation in tensor memory; nothing is dequantised).
 * Inputs: the rows grouped by expert and already quantised per row
 * (moe_quantize_nvfp4_rows with src_rows = sorted_rows, src_div = k):
 * x_codes [rows][H/2], x_sf [rows][H/16], x_G [rows]; offsets [E+1] (from
 * moe_permute).  Writes y_perm bf16 [rows][H]:
 *   g, u = (W_gate x, W_up x) * x_G * g_gu[e];  h = SiLU(g) * u   (fp32)
 *   h -> NVFP4 per row (as moe_quantize_nvfp4_rows);  y = (W_down h) * h_G * g_d[e]
 * Source: "Drama 3 - NVFP4 routed experts", section "Quantization" (NVFP4
 * weights and dynamic per-token activation scales), "drama-rs", "Layout"
 * (grouped MoE prefill).
 * Workspace: moe_prefill_nvfp4_workspace_bytes(rows, F) bytes, 256-byte
 * aligned: h fp32 [rows][F], then its codes [rows][F/2], scales [rows][F/16]
 * and globals [rows], each section starting on a 256-byte boundary.
 * Requirements: H % 256 == 0, F % 256 == 0, E <= 960, offsets as for
 * moe_ffn_grouped_prefill; x_codes, x_sf, y_perm 16-byte aligned.  rows == 0
 * is a no-op.
 */
MOE_API size_t moe_prefill_nvfp4_workspace_bytes(int rows, int F);
MOE_API moe_status moe_ffn_grouped_prefill_nvfp4(const moe_nvfp4_layer *layer,
                                                 const uint8_t *x_codes, const uint8_t *x_sf,
                                                 const float *x_G, const int32_t *offsets,
                                                 int rows, uint16_t *y_perm, void *ws,
                                                 size_t ws_bytes, moe_stream_t stream);

/*
 * Router-weighted combine: y[t] = sum over j = 0..k-1 (in that order) of
 * w[t][j] * Y[p(t*k + j)], accumulated in fp32 and rounded to nearest-even
 * bf16.  Y is y_rows (fp32, y_dtype 0) or y_perm (bf16, y_dtype 1), [T*k][H];
 * p = inv (from moe_permute) or the identity when inv is NULL.  Every output
 * row is owned by one thread block: no atomics, deterministic.
 * Requirements: H % 8 == 0.  T == 0 is a no-op.
 */
MOE_API moe_status moe_unpermute_combine(const void *Y, int y_dtype, const int32_t *inv,
                                         const float *w, int T, int k, int H, uint16_t *y,
                                         moe_stream_t stream);

/* ======================================================================== */
/* Device error word                                                         */
/* ======================================================================== */
/* Host pointer out receives (after a stream synchronise done by this call)
 * the device error word: 0 = none, otherwise a code naming the kernel and
 * wait that timed out.  The word is cleared on read. */
MOE_API moe_status moe_device_error(int *out, moe_stream_t stream);

/* Codes of the device error word. */
#define MOE_DEVERR_DECODE_H_WAIT 0x101 /* decode: a wait for h or a row output gave up */
#define MOE_DEVERR_DECODE_ROUTER_WAIT 0x102 /* decode with the router: a wait for a logit gave up */
#define MOE_DEVERR_PREFILL_WAIT 0x201  /* prefill: a pipeline barrier wait gave up */

/*
 * Test hooks for failure detection (no counterpart on the pages).  Each one
 * makes a bounded device-side wait run out on purpose, without any fault, so
 * that a test can check that the kernel gives up, returns, raises the device
 * error word and leaves the GPU usable:
 *   - moe_debug_starve_decode: moe_ffn_w4a16_decode whose gate/up work items
 *     consume their weights but publish no h, with the down items' wait for
 *     h bounded by `polls` polls (each >= 100 ns).  Raises
 *     MOE_DEVERR_DECODE_H_WAIT.  y_rows is left unspecified; zero-fill the
 *     workspace before its next use.
 *   - moe_debug_starve_prefill: the gate/up launch of moe_ffn_grouped_prefill
 *     whose weight producer issues no loads, every pipeline wait bounded by
 *     `polls` sleeping polls (each at most ~10 us).  Raises
 *     MOE_DEVERR_PREFILL_WAIT; the workspace (h) is left unspecified.
 * Arguments and errors as for the calls they derive from; polls >= 1.
 */
MOE_API moe_status moe_debug_starve_decode(const moe_w4_layer *layer, const uint16_t *x,
                                           const int32_t *idx, int T, int k, float *y_rows,
                                           void *ws, size_t ws_bytes, unsigned int polls,
                                           moe_stream_t stream);
MOE_API moe_status moe_debug_starve_prefill(const moe_w4_layer *layer, const uint16_t *x_perm,
                                            const int32_t *offsets, int rows, void *ws,
                                            size_t ws_bytes, unsigned int polls,
                                            moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
