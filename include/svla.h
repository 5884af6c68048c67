/*
 * svla.h — C ABI of libsvla: SmolVLA action-chunk generation on NVIDIA B200
 * (sm_100a).
 *
 * What the library computes ("noeira docs, SmolVLA" §Architecture; "Paper vs
 * hardware 11: SmolVLA" §claims):
 *   1. prefill: the SmolLM2 prefix LM (RMSNorm, GQA attention with RoPE,
 *      SwiGLU) runs once over the prefix embeddings and writes every layer's
 *      keys and values into a K/V cache;
 *   2. denoise: the action expert runs n_steps times; even layers do causal
 *      self-attention over the chunk, odd layers cross-attend to the cached
 *      K/V; a sinusoidal time embedding enters through the action-time MLP;
 *      each step applies x <- x + dt * v, dt = -1/n_steps, from Gaussian
 *      noise at t = 1 toward t = 0 (flow matching: x_t = t*eps + (1-t)*a).
 * Around that path: the prefix overwrite at a chunk junction
 * (svla_denoise_prefix), the prefix assembly from vision features
 * (svla_set_assembly / svla_assemble_prefix), the weight-only int8 prefix
 * (svla_create_ex with SVLA_CREATE_PREFIX_INT8), the expert's training step
 * (svla_train_step), and single kernels for callers that compose their own
 * schedule (svla_op_*).
 *
 * Conventions for every function below.
 *   - Pointers named "device" must point to memory of the handle's device
 *     (cudaMalloc'd, or a torch CUDA tensor's data_ptr). The library never
 *     frees caller memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). All device work is enqueued on it asynchronously; a call
 *     returns once the work is enqueued.
 *   - bf16 is IEEE bfloat16 stored as uint16; matrices are row-major.
 *   - Return value: SVLA_OK (0) or a negative svla_status. Argument and shape
 *     errors are detected on the host before anything is enqueued. Errors
 *     found on the device (a query with no valid prefix token, a bounded wait
 *     that ran out) are sticky in a per-device status word, reported by
 *     svla_device_status().
 *   - A handle may be used from one host thread at a time. Calls that use the
 *     same handle on different streams must not overlap in time on the GPU
 *     (they share the handle's workspace).
 */
#ifndef SVLA_H_
#define SVLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SVLA_API __attribute__((visibility("default")))
#else
#define SVLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int svla_status;
#define SVLA_OK                 0
#define SVLA_ERR_ARG           -1   /* null pointer, negative size, bad enum      */
#define SVLA_ERR_SHAPE         -2   /* size outside the handle's limits / layout  */
#define SVLA_ERR_BLOB_SIZE     -3   /* weight blob is not exactly the manifest    */
#define SVLA_ERR_EMPTY_PREFIX  -4   /* a query has no valid prefix token          */
#define SVLA_ERR_CUDA          -5   /* a CUDA runtime call failed                 */
#define SVLA_ERR_OOM           -6   /* device allocation failed                   */
#define SVLA_ERR_TIMEOUT       -7   /* a device-side bounded wait ran out         */
#define SVLA_ERR_UNSUPPORTED   -8   /* no sm_100 device                           */

typedef struct svla_handle svla_handle;

/* Model shape and handle limits. The SmolVLA instance is
 * {16, 960, 15, 5, 64, 2560, 16, 720, 15, 5, 2048, 32, 1e4, 1e-5, 4e-3, 4.0, ...}.
 * Constraints: head_dim in {32, 64}; p_heads % p_kv_heads == 0 and
 * e_heads % e_kv_heads == 0; p_layers == e_layers (expert layer l reads prefix
 * layer l's cache on odd l); every width a multiple of 64 except e_width,
 * action_dim (multiples of 8, action_dim <= 64) and p_ffn, e_ffn (multiples of 64). */
typedef struct svla_config {
  int p_layers, p_width, p_heads, p_kv_heads, head_dim, p_ffn;
  int e_layers, e_width, e_heads, e_kv_heads, e_ffn, action_dim;
  float rope_base, rms_eps, t_min_period, t_max_period;
  int max_batch, max_prefix, max_chunk;
} svla_config;

/* Create a handle on `device` from a flat weight blob.
 *   blob: bf16, host or device memory, the weights in manifest order —
 *     per prefix layer l: in_norm[D], wq[nq*hd, D], wk[nkv*hd, D], wv[nkv*hd, D],
 *       wo[D, nq*hd], post_norm[D], wg[F, D], wu[F, D], wd[D, F];
 *     per expert layer l: in_norm[E], wq[eq*hd, E], wk[ekv*hd, X], wv[ekv*hd, X]
 *       (X = E on even l, X = nkv*hd on odd l: the cross projection of the
 *       cached prefix K/V), wo[E, eq*hd], post_norm[E], wg[Fe, E], wu[Fe, E], wd[E, Fe];
 *     then final_norm[E], w_in[E, A], b_in[E], w_t1[E, 2E], b_t1[E], w_t2[E, E],
 *       b_t2[E], w_out[A, E], b_out[A].
 *     Matrices are [out, in] as nn.Linear stores them ("noeira docs, SmolVLA"
 *     §Weights). The blob is copied; the caller may free it on return.
 *   blob_bytes must equal the manifest total, else SVLA_ERR_BLOB_SIZE.
 * Allocates the weights, a workspace sized by max_batch/max_prefix/max_chunk
 * and small tables; *out receives the handle (NULL on error). */
SVLA_API svla_status svla_create(const svla_config* cfg, const void* blob, size_t blob_bytes,
                        int device, svla_handle** out);

/* svla_create with options. flags is a bitwise OR of:
 *   SVLA_CREATE_PREFIX_INT8  also build the weight-only int8 copy of the prefix
 *     LM's projections (the "vlm-8bit" preset of the mlx-smolvla PyPI page,
 *     §Run a checkpoint) and select it for svla_prefill; the dense bf16
 *     weights stay resident, so svla_set_prefix_weights can switch back.
 *     Scheme (the page names the preset only; these are readings): every group
 *     of 64 consecutive input weights of one output row of W_q, W_k, W_v, W_o,
 *     W_g, W_u, W_d gets lo = min, hi = max, alpha = bf16((hi - lo) / 255),
 *     beta = lo and codes q = clamp(rint((w - beta) / alpha), 0, 255) (0 when
 *     alpha = 0), each step an IEEE fp32 operation rounded to nearest even; the
 *     GEMMs use w^ = bf16(alpha q + beta) (times the folded RMSNorm gain, as the
 *     dense path does). Norm gains, the expert and the heads stay bf16.
 *     Needs p_width and p_ffn multiples of 64 (they are, by check_config).
 * flags = 0 is svla_create. Unknown flag bits: SVLA_ERR_ARG. */
#define SVLA_CREATE_PREFIX_INT8 1u
/*   SVLA_CREATE_TRAIN  also keep the expert and head weights as given (no
 *     folding or interleaving) and allocate the workspace of svla_train_step
 *     for max_batch x max_chunk rows (every expert layer's activations are
 *     kept for the backward: about 0.55 MB per row at the SmolVLA shape). */
#define SVLA_CREATE_TRAIN 2u
/*   SVLA_CREATE_EXPERT_INT8  also build the weight-only int8 copy of the action
 *     expert's projections and select it for svla_denoise / svla_sample (the
 *     same scheme as SVLA_CREATE_PREFIX_INT8, on W_q, W_k, W_v, W_o, W_g, W_u,
 *     W_d of every expert layer, the odd layers' cross W_k / W_v included; the
 *     expert's 720-wide inputs are not a multiple of 64, so the last group of a
 *     row holds its K mod 64 remaining inputs). The heads (action_in, the time
 *     MLP, action_out) and the norm gains stay bf16; the dense weights stay
 *     resident, so svla_set_expert_weights can switch back. Both denoise paths
 *     read the codes: the persistent kernel dequantises each weight slice in
 *     shared memory, the multi-kernel path uses the int8 GEMM (few tiles) or a
 *     per-matrix dequantisation before the dense GEMM (many tiles). */
#define SVLA_CREATE_EXPERT_INT8 4u
SVLA_API svla_status svla_create_ex(const svla_config* cfg, const void* blob, size_t blob_bytes,
                           int device, unsigned flags, svla_handle** out);

/* Prefix weights svla_prefill uses from the next call on: 16 = dense bf16
 * (default), 8 = the int8 copy (SVLA_ERR_UNSUPPORTED unless the handle was
 * created with SVLA_CREATE_PREFIX_INT8). Other values: SVLA_ERR_ARG. */
SVLA_API svla_status svla_set_prefix_weights(svla_handle* h, int bits);
/* The prefix weight width svla_prefill uses (16 or 8); 0 for a NULL handle. */
SVLA_API int svla_prefix_weights(const svla_handle* h);

/* Expert weights svla_denoise, svla_denoise_prefix and svla_sample use from
 * the next call on: 16 = dense bf16 (default), 8 = the int8 copy
 * (SVLA_ERR_UNSUPPORTED unless the handle was created with
 * SVLA_CREATE_EXPERT_INT8). Other values: SVLA_ERR_ARG. */
SVLA_API svla_status svla_set_expert_weights(svla_handle* h, int bits);
/* The expert weight width the denoise uses (16 or 8); 0 for a NULL handle. */
SVLA_API int svla_expert_weights(const svla_handle* h);

/* Training step of the action expert ("noeira docs, SmolVLA" §Architecture,
 * the fine-tune's flow-matching objective; §Fine-tuning: the 16 expert layers
 * and the action and time projections train, the language model is frozen).
 * Readings: x_t = t_b eps + (1 - t_b) a per query, v = v(x_t, t_b | prefix),
 * loss = mean over the B H A terms of (v - (eps - a))^2; the result is the loss
 * and its gradient with respect to every expert and head tensor (no optimiser
 * update).
 *   kv_cache, pad_mask: the frozen prefix, as for svla_denoise (device).
 *   actions: the target chunk a, noise: eps, device float32 [B, H, A];
 *   t: device float32 [B], the flow time of each query.
 *   loss: device float32 scalar (written).
 *   grads: device float32, svla_train_grad_elems(h) elements, 16-byte aligned:
 *     every tensor of the blob from the first expert layer's in_norm to b_out,
 *     in manifest order and shape ([out, in] for matrices) (written in full).
 * The forward uses the weights given to svla_create_ex; work is stream-ordered
 * and bitwise reproducible (fixed-order reductions). The step runs as one CUDA
 * graph, captured on the first call with a given (B, L, H, buffers) and
 * replayed afterwards (like svla_denoise), so make that first call before
 * any stream capture of your own. Needs a handle created
 * with SVLA_CREATE_TRAIN (else SVLA_ERR_UNSUPPORTED); B, L, H within the
 * handle's limits (else SVLA_ERR_SHAPE). */
SVLA_API svla_status svla_train_step(svla_handle* h, const void* kv_cache, const uint8_t* pad_mask, int B,
                            int L, const float* actions, const float* noise, const float* t, int H,
                            float* loss, float* grads, void* stream);
/* Number of float32 gradient elements of svla_train_step (0 without a training workspace). */
SVLA_API size_t svla_train_grad_elems(const svla_handle* h);

/* Free everything the handle owns (synchronises its device first). NULL is ok. */
SVLA_API svla_status svla_destroy(svla_handle* h);

/* Exact byte size of a K/V cache for B queries of L prefix tokens:
 * K block then V block, each [p_layers][B][L][p_kv_heads*head_dim] bf16
 * (token-major; K after RoPE). 0 on bad arguments. */
SVLA_API size_t svla_kv_cache_bytes(const svla_handle* h, int B, int L);

/* Bytes of the blob the handle expects (the manifest total). */
SVLA_API size_t svla_blob_bytes(const svla_config* cfg);

/* Prefix prefill ("noeira docs, SmolVLA" §Architecture: the VLM runs once over
 * the prefix and caches its keys and values).
 *   prefix_embeds: device bf16 [B, L, p_width].
 *   pad_mask:      device uint8 [B, L], 1 = real token, 0 = padding (anywhere).
 *                  Positions are cumsum(valid) - 1; a query with no valid token
 *                  sets SVLA_ERR_EMPTY_PREFIX in the device status.
 *   kv_cache:      device, svla_kv_cache_bytes(h, B, L) bytes, written in full
 *                  except that pad slots hold values readers must mask.
 * 1 <= B <= max_batch, 1 <= L <= max_prefix. */
SVLA_API svla_status svla_prefill(svla_handle* h, const void* prefix_embeds, const uint8_t* pad_mask,
                         int B, int L, void* kv_cache, void* stream);

/* Euler flow-matching denoise of the action chunk ("noeira docs, SmolVLA"
 * §Architecture: from Gaussian noise at t = 1, each of the steps predicts a
 * velocity and moves toward t = 0).
 *   kv_cache, pad_mask: as written / read by svla_prefill (same B, L).
 *   noise:   device float32 [B, H, action_dim], x at t = 1.
 *   actions: device float32 [B, H, action_dim], receives x after n_steps (may
 *            alias noise).
 *   trace:   NULL, or device float32 [n_steps][2][B][H][action_dim]: per step k
 *            the velocity v_k at (x_k, t_k) and the state x_{k+1}.
 * 1 <= H <= max_chunk, 1 <= n_steps <= 1000. The whole loop (the hoisted cross
 * K/V projection and every step) is replayed from one CUDA graph per shape and
 * buffer set. */
SVLA_API svla_status svla_denoise(svla_handle* h, const void* kv_cache, const uint8_t* pad_mask,
                         int B, int L, const float* noise, int H, int n_steps,
                         float* actions, float* trace, void* stream);

/* svla_denoise with the gradient-free prefix overwrite at a chunk junction
 * ("Paper vs hardware 11: SmolVLA" §What I ran: the actions that run during
 * the inference delay are taken from the previous chunk, which removes most of
 * the jump at the handover). After every Euler step the first d rows of each
 * query's state are set to t·noise + (1 − t)·prefix, t the time reached, so
 * the chunk is denoised conditioned on them and ends with exactly `prefix`.
 *   prefix: device float32 [B, d, action_dim]; 0 <= d <= H (d = 0: svla_denoise).
 *   actions must not alias noise when d > 0 (the overwrite reads the noise).
 * Other arguments as svla_denoise; the trace holds the overwritten states. */
SVLA_API svla_status svla_denoise_prefix(svla_handle* h, const void* kv_cache, const uint8_t* pad_mask,
                                         int B, int L, const float* noise, int H, int n_steps,
                                         const float* prefix, int d, float* actions, float* trace,
                                         void* stream);

/* Which implementation runs the denoise of svla_denoise, svla_denoise_prefix
 * and svla_sample on this handle. Both compute the same path (same readings,
 * same bf16 rounding points); each is bitwise run-to-run deterministic and both
 * meet the parity tolerances, but they round in different orders, so their
 * results differ in the last bits.
 *   SVLA_DENOISE_AUTO   (default) FUSED when svla_denoise_fused_supported, else GRAPH.
 *   SVLA_DENOISE_GRAPH  one CUDA graph: the hoisted cross K/V projection, then
 *                       ~85 dependent kernels per Euler step; any shape.
 *   SVLA_DENOISE_FUSED  the hoisted projection, then ONE persistent kernel for
 *                       all steps (one CTA per SM, cooperative launch, the
 *                       dependent steps as stages separated by grid barriers);
 *                       needs B * H <= 64 and H <= 64, else the denoise call
 *                       returns SVLA_ERR_UNSUPPORTED.
 * Returns SVLA_ERR_ARG for another value or a null handle. */
#define SVLA_DENOISE_AUTO   0
#define SVLA_DENOISE_GRAPH  1
#define SVLA_DENOISE_FUSED  2
SVLA_API svla_status svla_set_denoise_path(svla_handle* h, int path);

/* 1 if the persistent denoise kernel takes batch B with chunk length H on
 * this handle for every prefix length up to max_prefix (B * H <= 64, H <= 64,
 * within the handle's limits, and a head's prefix keys and values fit in
 * shared memory), else 0. */
SVLA_API int svla_denoise_fused_supported(const svla_handle* h, int B, int H);

/* Draw the noise, prefill, denoise, on one stream.
 * Noise: Philox4x32-10 keyed by seed (key = {seed low 32, seed high 32}),
 * counter {block, query, 0, 0}; element e of a query's [H, A] noise is lane
 * e % 4 of block e / 4; Box–Muller on the pairs (r0, r1) and (r2, r3) with
 * u1 = ((r >> 8) + 1) / 2^24, u2 = (r >> 8) / 2^24.
 *   kv_cache: device buffer as for svla_prefill (written).
 *   noise_out: NULL or device float32 [B, H, A] receiving the drawn noise. */
SVLA_API svla_status svla_sample(svla_handle* h, const void* prefix_embeds, const uint8_t* pad_mask,
                        int B, int L, uint64_t seed, int H, int n_steps,
                        void* kv_cache, float* noise_out, float* actions, void* stream);

/* Prefix assembly upstream of the prefill ("noeira docs, SmolVLA"
 * §Architecture: the connector — pixel shuffle of the vision tower's patch
 * grid, then a linear projection to the LM width — and a prefix of the camera
 * images, the tokenised instruction and one state token; "Paper vs hardware
 * 11: SmolVLA" §claims: the state projected to one token). Pixel shuffle x r
 * is the space-to-depth of the g x g patch grid: output token (i, j)
 * concatenates the r x r block of patches (r i + a, r j + b) in row-major
 * (a, b) order; the state token is W_s s + b_s in fp32, stored bf16; the
 * prefix is [image tokens in camera order | text tokens | state token].
 *
 * svla_set_assembly: blob = bf16 [W_c (p_width x r*r*vis_width) | W_s
 *   (p_width x state_dim) | b_s (p_width)], host or device memory, copied
 *   (svla_assembly_blob_bytes gives its size; another size is
 *   SVLA_ERR_BLOB_SIZE). vis_width a multiple of 8, grid a multiple of
 *   shuffle, 1 <= state_dim <= 64; allocates the workspace for max_batch x
 *   max_images images. Call once, outside any stream capture.
 * svla_assemble_prefix: vis device bf16 [B][n_img][grid*grid][vis_width]
 *   (row-major patch index); text device bf16 [B][T][p_width] with text_valid
 *   device u8 [B][T] (both may be NULL when T = 0); state device f32
 *   [B][state_dim]; writes embeds device bf16 [B][L][p_width] and pad device
 *   u8 [B][L], L = n_img (grid/shuffle)^2 + T + 1 — the inputs of
 *   svla_prefill. Stream-ordered; 1 <= B <= max_batch, 1 <= n_img <=
 *   max_images. */
SVLA_API size_t svla_assembly_blob_bytes(int p_width, int vis_width, int shuffle, int state_dim);
SVLA_API svla_status svla_set_assembly(svla_handle* h, const void* blob, size_t blob_bytes, int vis_width,
                                       int grid, int shuffle, int state_dim, int max_images);
SVLA_API svla_status svla_assemble_prefix(svla_handle* h, const void* vis, const void* text,
                                          const uint8_t* text_valid, const float* state, int B, int n_img,
                                          int T, void* embeds, uint8_t* pad, void* stream);

/* Synchronise `stream`, then return and clear the device status word of the
 * handle's device (SVLA_OK, SVLA_ERR_EMPTY_PREFIX, SVLA_ERR_TIMEOUT) — or
 * SVLA_ERR_CUDA if the synchronisation itself failed. */
SVLA_API svla_status svla_device_status(svla_handle* h, void* stream);

/* Text of the last error set on this handle (or, for h == NULL, by the last
 * failing call of this thread). Never NULL. */
SVLA_API const char* svla_last_error(const svla_handle* h);
SVLA_API const char* svla_status_string(svla_status s);

/* ---------------------------------------------------------------------------
 * Kernel-level entry points (no handle). They expose single kernels of the
 * path so each can be checked on its own; they use the same code as the path.
 * ------------------------------------------------------------------------- */

/* Epilogues of svla_op_gemm. */
#define SVLA_EPI_F32        0   /* C(f32)  = acc (+ bias)                     */
#define SVLA_EPI_BF16       1   /* C(bf16) = acc (+ bias)                     */
#define SVLA_EPI_ADD_F32    2   /* C(f32) += acc (+ bias)    (residual add)   */
#define SVLA_EPI_SILU_BF16  3   /* C(bf16) = silu(acc + bias)                 */

/* C[M, N] = A[M, K] · W[N, K]^T on the tcgen05 tensor cores, bf16 inputs,
 * fp32 accumulation (the projections of every layer: "noeira docs, SmolVLA"
 * §Architecture, nn.Linear [out, in] weights).
 *   A: device bf16, row stride lda >= K elements; W: device bf16, row stride
 *   ldw >= K; C: device, row stride ldc >= N (f32 or bf16 per epilogue);
 *   bias: NULL or device float32 [N].
 *   Strides must be multiples of 8 elements and pointers 16-byte aligned (TMA).
 *   splits: K-split count (0 = choose); with splits > 1 partial tiles go to
 *   `workspace` (device, >= svla_op_gemm_workspace_bytes(M, N, K, splits)
 *   bytes, its counter area zeroed once before first use and left zeroed by
 *   every call) and the last CTA of each tile sums them in fixed order, so the
 *   result is bitwise deterministic.
 *   status: device int, set (first error wins) to SVLA_ERR_TIMEOUT if a
 *   bounded wait ran out; may be NULL. */
SVLA_API svla_status svla_op_gemm(int epilogue, const void* A, int lda, const void* W, int ldw,
                         int M, int N, int K, void* C, int ldc, const float* bias,
                         int splits, void* workspace, size_t workspace_bytes,
                         int* status, void* stream);
SVLA_API size_t svla_op_gemm_workspace_bytes(int M, int N, int K, int splits);
/* The K-split count svla_op_gemm picks for splits = 0. */
SVLA_API int svla_op_gemm_splits(int M, int N, int K);

/* GQA attention (readings 1, 4–7): out = softmax(q k^T / sqrt(hd) + mask) v.
 *   q: device bf16 [B, Lq, n_q*hd] (row stride ldq), k/v: device bf16
 *   [B, Lk, n_kv*hd] (row stride ldkv); out: device bf16 [B, Lq, n_q*hd]
 *   (row stride ldo). key_valid: NULL (all valid) or device uint8 [B, Lk].
 *   causal: key j visible to row i only if j <= i. Query head h reads kv head
 *   h / (n_q / n_kv). hd in {32, 64}. Every row needs >= 1 visible key. */
SVLA_API svla_status svla_op_attention(const void* q, int ldq, const void* k, const void* v, int ldkv,
                              const uint8_t* key_valid, int B, int n_q, int n_kv, int hd,
                              int Lq, int Lk, int causal, void* out, int ldo, void* stream);

/* The int8 quantiser of the vlm-8bit and expert presets (svla_create_ex,
 * SVLA_CREATE_PREFIX_INT8 / SVLA_CREATE_EXPERT_INT8) on one matrix: groups of
 * 64 consecutive inputs of a row, the last group holding the K mod 64
 * remaining inputs where K % 64 != 0 (mlx-smolvla PyPI page, §Run a checkpoint,
 * for the scheme's name; the group rules are this library's readings).
 *   W:  device bf16 [N, K], row stride ldw >= K elements (even), 4-byte aligned.
 *   q:  device uint8 [N, K] codes, row stride ldq >= K bytes (even).
 *   ab: device bf16 [G][N][2], G = ceil(K/64): (alpha, beta) of row n, group g at (g, n).
 *   K % 16 == 0, N >= 1; weights must be finite. Asynchronous on `stream`. */
SVLA_API svla_status svla_op_quantize_affine8(const void* W, int ldw, int N, int K, void* q, int ldq,
                                     void* ab, void* stream);

/* C[M, N] = A[M, K] · W^[N, K]^T with W^[n, k] = bf16(bf16(alpha q + beta) * g[k])
 * on the tcgen05 tensor cores (the int8 weights are dequantised in shared
 * memory, fp32 accumulation). Epilogues and C as svla_op_gemm.
 *   A: device bf16, row stride lda >= K (multiple of 8), 16-byte aligned.
 *   q, ab: as written by svla_op_quantize_affine8 (ldq a multiple of 16).
 *   gain: NULL (g = 1) or device bf16 [K], 16-byte aligned.
 *   K % 16 == 0, N % 8 == 0. splits: 0 = choose, else 1..8 (cluster split-K;
 *   no workspace). status: as svla_op_gemm. */
SVLA_API svla_status svla_op_gemm_w8(int epilogue, const void* A, int lda, const void* q, int ldq,
                            const void* ab, const void* gain, int M, int N, int K, void* C, int ldc,
                            const float* bias, int splits, int* status, void* stream);
/* The K-split count svla_op_gemm_w8 picks for splits = 0, and its tile width. */
SVLA_API int svla_op_gemm_w8_splits(int M, int N, int K);
SVLA_API int svla_op_gemm_w8_tile_n(int M, int N, int K);

/* RMSNorm (reading 8): y(bf16)[M, D] = x(f32)[M, D] / sqrt(mean(x^2) + eps) * g(bf16)[D]. */
SVLA_API svla_status svla_op_rmsnorm(const float* x, const void* g, int M, int D, float eps,
                            void* y, void* stream);

/* svla_op_gemm without a workspace argument, for callers that cannot allocate
 * GPU memory themselves: code that must not call cudaMalloc once it is running
 * (a robot control loop that forbids allocation after start-up because its
 * latency is unpredictable), a host that owns all device memory through its
 * own pool, or a plain-C caller with no allocator of its own. This entry point
 * has no counterpart in the paper; it exists only for these callers.
 *   Same arguments and results as svla_op_gemm, minus the workspace. The
 *   split-K scratch is a fixed device array of SVLA_NOALLOC_SCRATCH_BYTES
 *   (8 MiB) in the library, present on every GPU that loads it until the
 *   process exits. A GEMM whose plan needs more scratch than that
 *   (svla_op_gemm_workspace_bytes(M, N, K, splits) > 8 MiB) is rejected with
 *   SVLA_ERR_SHAPE and a message naming both sizes; nothing is launched.
 *   The first call on a device resolves the array's device address and zeroes
 *   its 4 KiB counter area synchronously, so make that first call before any
 *   stream capture. The address is kept for the life of the process: do not
 *   call this entry point after cudaDeviceReset. Each call that splits K
 *   clears the counter area on `stream` before its launch; a plan whose
 *   counters would not fit in it is rejected with SVLA_ERR_SHAPE. The
 *   function never calls cudaMalloc, cudaFree or any allocating library
 *   routine.
 *   All calls on a device share the one scratch array: calls whose kernels
 *   overlap on the GPU (different streams, or several host threads) race and
 *   may give wrong results; issue them in one stream order. */
#define SVLA_NOALLOC_SCRATCH_BYTES (8u << 20)
SVLA_API svla_status svla_op_gemm_noalloc(int epilogue, const void* A, int lda, const void* W, int ldw,
                                          int M, int N, int K, void* C, int ldc, const float* bias,
                                          int splits, int* status, void* stream);

/* Set the limit, in nanoseconds, of every device-side bounded wait of later
 * launches (default 1e9). A limit of 0 makes any wait that is not already
 * satisfied give up at once and report SVLA_ERR_TIMEOUT; it exists to test
 * that path. Process-wide. */
SVLA_API void svla_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* SVLA_H_ */
