/*
 * uno.h — C ABI of the sm_100a (B200) Psi-Spec linear decode step.
 *
 * The method ("Uno", diffusion-augmented LLMs with the Psi-Spec sampler):
 *   - every AR weight matrix carries a LoRA adapter theta_Delta; drafting uses
 *     theta_AR + theta_Delta, verification theta_AR alone (hyper.ai page,
 *     section "方法", the paragraph on theta_Delta);
 *   - one forward serves both paths through a per-row gate that switches the
 *     adapter off on clean rows and on for noisy rows (same section, the
 *     gated-LoRA paragraph; ainews page: "conditional LoRA");
 *   - the linear sampler drafts one block from the draft path's per-position
 *     marginals, and rejection sampling against the AR distribution keeps the
 *     longest accepted prefix (same section, the Psi-Spec paragraph);
 *   - "lossless" means the output follows the AR distribution (ainews page).
 *
 * Conventions for every call
 *   - Pointers named as device pointers must be device memory of the current
 *     device, 16-byte aligned. The caller owns every buffer; the library never
 *     allocates device memory on these calls (scratch comes from `workspace`,
 *     sized by the matching *_workspace query).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls
 *     only enqueue work on it and return; results are ready when the stream
 *     reaches them.
 *   - Errors found on the host return a status at once and launch nothing;
 *     uno_last_error() describes the last one on the calling thread.
 *     Conditions found on the device (a draft id outside the vocabulary, a NaN
 *     logit, a bounded wait that gave up) OR bits into `dev_status` (where the
 *     call has one) and into the library's device status word (see
 *     uno_device_status); no kernel traps.
 *   - Row-major layouts throughout. bf16 is IEEE bfloat16 bits; f32 is float.
 */
#ifndef UNO_H_
#define UNO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  UNO_OK = 0,
  UNO_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or value */
  UNO_ERR_UNSUPPORTED = 2,  /* valid but outside the supported range */
  UNO_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  UNO_ERR_TIMEOUT = 4,      /* reported through uno_device_status */
  UNO_ERR_DEVICE_FLAG = 5,  /* reported through uno_device_status */
  UNO_ERR_WORKSPACE = 6     /* workspace NULL or smaller than the query says */
} uno_status;

typedef enum { UNO_BF16 = 0, UNO_F32 = 1 } uno_dtype;

/* Device status bits (dev_status words and uno_device_status). */
#define UNO_DEV_BAD_DRAFT 1 /* a draft id outside [0, V): that sequence's outputs are -1 */
#define UNO_DEV_NAN 2       /* a NaN logit in a row that was read: outputs are -1 */
#define UNO_DEV_TIMEOUT 4   /* a bounded on-device wait gave up (kernel returned early) */

/* Message for the last failed call on this thread (static storage, valid
 * until the next call on this thread). Never NULL. */
const char* uno_last_error(void);

/* Library version string. */
const char* uno_version(void);

/* Read the library-wide device status word of the current device into
 * *bits_out (synchronises `stream`), clearing it when `clear` != 0. */
uno_status uno_device_status(int32_t* bits_out, int32_t clear, void* stream);

/* ---------------------------------------------------------------------------
 * Gated-LoRA linear (hyper.ai page, section "方法": LoRA adapter on every AR
 * matrix, gated per row in one forward pass):
 *
 *     y = x W^T + scale * g (.) ((x A^T) Bl^T)
 *
 *   x [M,K], W [N,K], A [r,K], Bl [N,r] (nn.Linear / PEFT layout), all `dt`;
 *   gate [M] uint8 in {0,1} (0 = adapter off: the verify path theta_AR;
 *   1 = adapter on: the draft path theta_AR + theta_Delta); y [M,N] `dt`.
 *   fp32 accumulation. The rank-r product x A^T is rounded to `dt` before the
 *   up-projection, which runs in the same tensor-core pass as x W^T, so W is
 *   read from HBM once. Decode-size bf16 batches (M <= 128, r <= 128) run in
 *   one launch that splits K into slices and rounds each slice's x_s A_s^T.
 *   Sizes: M >= 0 (M = 0 launches nothing), K >= 1, N >= 1, 0 <= r <= 256.
 *   bf16: K, N, r multiples of 8; f32: multiples of 4 (16-byte row strides).
 *   f32 inputs run on the tf32 tensor-core path (10-bit mantissa products).
 *   workspace: >= uno_gated_lora_linear_workspace(...) bytes of device
 *   memory, 16-byte aligned, any contents; required when r > 0. When r = 0 it
 *   may be NULL (or smaller than the query): the call then runs without the
 *   scratch below. bf16 batches with M > 256 (the CTA-pair kernel) also keep
 *   in it the fp32 partial sums of tiles whose K range two pairs of SMs share
 *   (stream-K over the last round of tiles) and the flags that order them;
 *   the call clears those flags on `stream` before the pairs use them.
 *   Calls that share a workspace must not run at the same time.
 * ------------------------------------------------------------------------- */
size_t uno_gated_lora_linear_workspace(uno_dtype dt, int64_t M, int64_t K, int64_t N, int32_t r);

uno_status uno_gated_lora_linear(uno_dtype dt, int64_t M, int64_t K, int64_t N, int32_t r,
                                 const void* x, const void* W, const void* A, const void* Bl,
                                 const uint8_t* gate, float scale, void* y, void* workspace,
                                 size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Gradients of the gated-LoRA adapter, the AR weights frozen (hyper.ai page,
 * section "方法", the training-order paragraph: the AR weights stay fixed
 * while the diffusion adapter trains). For the linear above and an output
 * gradient dy [M,N], with t_u = x A^T:
 *
 *     dBl = (scale * g (.) dy)^T t_u      [N, r]
 *     dA  = (dy Bl)^T (scale * g (.) x)   [r, K]
 *
 *   x [M,K], dy [M,N], A [r,K], Bl [N,r], gate [M] uint8: bf16 (the only
 *   dtype); dA [r,K] and dBl [N,r] bf16 outputs. fp32 accumulation; t_u and
 *   dy Bl are rounded to bf16 (tensor-core operands). Gate-0 rows contribute
 *   nothing. Sizes: K, N multiples of 8, 8 <= r <= 256 (multiple of 8),
 *   M >= 0 (M = 0 writes zero gradients). workspace: >=
 *   uno_gated_lora_backward_workspace(M, K, N, r) bytes, 16-byte aligned, any
 *   contents (x and dy transposed, and the rank-r products).
 * ------------------------------------------------------------------------- */
size_t uno_gated_lora_backward_workspace(int64_t M, int64_t K, int64_t N, int32_t r);

uno_status uno_gated_lora_backward(uno_dtype dt, int64_t M, int64_t K, int64_t N, int32_t r,
                                   const void* x, const void* dy, const void* A, const void* Bl,
                                   const uint8_t* gate, float scale, void* dA, void* dBl,
                                   void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Grouped gated-LoRA linears sharing one input x [M,K] (one launch for the
 * down-projections, one for the products; hyper.ai page, section "方法": the
 * adapter is attached to every AR matrix, so the q, k, v projections of a
 * layer, or its gate and up projections, read the same gated input):
 *
 *   mode 0:  y[i] = x W[i]^T + scale * g (.) ((x A[i]^T) Bl[i]^T),  i < G
 *   mode 1:  G = 2, N[0] = N[1]:  y[0] = silu(lin_0(x)) * lin_1(x)   (silu(a) = a/(1+e^-a))
 *
 *   W[i] [N[i],K], A[i] [r,K], Bl[i] [N[i],r], y[i] [M,N[i]], all `dt`
 *   (mode 1: bf16 only); gate [M] uint8; 1 <= G <= 3. Sizes as for
 *   uno_gated_lora_linear. workspace: >= uno_gated_lora_linear_group_workspace.
 * ------------------------------------------------------------------------- */
size_t uno_gated_lora_linear_group_workspace(uno_dtype dt, int64_t M, int32_t r, int32_t G);

uno_status uno_gated_lora_linear_group(uno_dtype dt, int64_t M, int64_t K, int32_t r, int32_t G,
                                       const int64_t* N, const void* x, const void* const* W,
                                       const void* const* A, const void* const* Bl,
                                       const uint8_t* gate, float scale, int32_t mode,
                                       void* const* y, void* workspace, size_t ws_bytes,
                                       void* stream);

/* ---------------------------------------------------------------------------
 * Psi-Spec verification of one drafted block per sequence (hyper.ai page,
 * section "方法", the Psi-Spec paragraph: rejection sampling against the base
 * AR distribution, longest valid prefix; ainews page: lossless).
 *
 *   p_logits [B,k_p,V]: AR logits for the k drafted positions (k_p = k) plus,
 *     when k_p = k+1, the position after the block (bonus draw).
 *   q_logits [B,k,V]: draft logits; draft [B,k] int32: the drafted ids.
 *   With p = softmax(p_logits / T), q = softmax(q_logits / T) per position
 *   and uniforms u from Philox4x32-10 (counter = (b_global*k + j, step lo,
 *   step hi, stream), key = (seed lo, seed hi), u = (word0 >> 8) * 2^-24,
 *   b_global = seq_offset + b; stream 1 accept, 2 residual, 3 bonus):
 *     accept position j iff u1 * q_j(d_j) < p_j(d_j);
 *     n = first rejected position (k if none)          -> accepted_len[b]
 *     out_tokens[b] = d_0..d_{n-1}, then
 *       if n < k: r = smallest v with C(v) > u2 * C(V-1), C the inclusive
 *                 cumulative sum of max(p_n - q_n, 0) in ascending id (p_n
 *                 itself if that sum is 0);
 *       if n = k and k_p = k+1: the bonus, same rule on p_k with u3;
 *     padded with -1; out_count[b] = number of tokens written.
 *   out_tokens is [B, k+1]. T > 0. 1 <= k <= 32, 2 <= V <= 196608.
 *   dev_status: optional int32 device word, OR-ed with UNO_DEV_* bits.
 * ------------------------------------------------------------------------- */
size_t uno_psi_verify_workspace(int32_t B, int32_t k, int32_t k_p, int32_t V);

uno_status uno_psi_verify(uno_dtype dt, int32_t B, int32_t k, int32_t k_p, int32_t V,
                          const void* p_logits, const void* q_logits, const int32_t* draft,
                          float temperature, uint64_t seed, uint64_t step, uint64_t seq_offset,
                          int32_t* accepted_len, int32_t* out_tokens, int32_t* out_count,
                          int32_t* dev_status, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * uno_psi_verify without a workspace: a library addition, the pages have no
 * counterpart. For callers that cannot allocate device memory where they
 * verify (cudaMalloc/cudaFree may synchronise the whole device and stall a
 * decode loop; some host runtimes own no device allocator).
 *
 *   Arguments, checks, kernels and results: those of uno_psi_verify, with the
 *   stats scratch taken from a 2 MiB static device array inside the library
 *   (one per device) instead of a workspace.
 *   Limit: uno_psi_verify_workspace(B, k, k_p, V) <= 2 MiB, which holds
 *     B * (k_p + k) <= 262144 logit rows; larger calls return
 *     UNO_ERR_UNSUPPORTED and launch nothing.
 *   Setup: the first call on a device (the current device, which must own
 *     the buffers and the stream) looks up the array's device address, which
 *     may load the library's module; make that first call before any stream
 *     capture begins. Later calls do no setup and reuse that address, so a
 *     device reset (cudaDeviceReset, or the primary context destroyed and
 *     created again) leaves it stale: do not call this entry point on that
 *     device again in the same process after one.
 *   Starting values: none needed; every entry a call reads it wrote itself.
 *   Concurrency: all calls on one device share the array. Calls on one stream
 *     are ordered and safe; calls whose kernels may overlap (other streams
 *     without ordering, other host threads) race on it and give wrong results.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * ------------------------------------------------------------------------- */
uno_status uno_psi_verify_noalloc(uno_dtype dt, int32_t B, int32_t k, int32_t k_p, int32_t V,
                                  const void* p_logits, const void* q_logits,
                                  const int32_t* draft, float temperature, uint64_t seed,
                                  uint64_t step, uint64_t seq_offset, int32_t* accepted_len,
                                  int32_t* out_tokens, int32_t* out_count, int32_t* dev_status,
                                  void* stream);

/* ---------------------------------------------------------------------------
 * Tree-sampler verification (hyper.ai page, section "方法": at low batch
 * sizes several candidate blocks are drawn and verified at once as a prefix
 * tree; lossless as the linear sampler). Per sequence b:
 *   cands [B,N,k] int32: N candidate blocks, each drawn from the per-position
 *     draft marginals (N independent linear-sampler blocks).
 *   The trie of the candidates is numbered in order of first visit when the
 *     candidates are walked from the root in index order; node 0 is the root.
 *     p_logits [B,R,V] `dt`: row n holds the AR logits of the next token after
 *     node n's prefix (row 0: the anchor's). R >= the node count (at most
 *     N*k + 1); rows of depth-k nodes are read only when `bonus` != 0.
 *   q_logits [B,k,V] `dt`: the draft logits of position j.
 *   At a node of depth j the live candidates (prefix = accepted path) are
 *   tested in index order: candidate i with token x is accepted iff
 *   u1 * q_j(x) < r_i(x), u1 from Philox stream 1 at index
 *   ((seq_offset + b)*k + j)*N + i, r_1 = softmax(p_logits[b,node] / T) and,
 *   after each rejection, r_{i+1} = max(r_i - q_j, 0) normalised (unchanged
 *   when its mass is 0). On acceptance the walk moves to the child with every
 *   candidate holding that token; if all are rejected, a token is drawn from
 *   the last residual (stream 2, index (seq_offset + b)*k + j) and the block
 *   ends. With all k accepted and `bonus` != 0, a bonus token is drawn from
 *   the leaf's AR row (stream 3, index (seq_offset + b)*k + k).
 *   Outputs as uno_psi_verify: accepted_len [B], out_tokens [B,k+1] (-1
 *   padded), out_count [B]. With N = 1 the results equal uno_psi_verify's
 *   (k_p = k, or k + 1 with the bonus).
 *   Sizes: 1 <= N <= 32, 1 <= k <= 32, 1 <= R <= N*k + 1, V as for
 *   uno_psi_verify; B * (R + k) <= 2^30; (seq_offset + B) * (k + 1) * N <= 2^32.
 *   Device-detected: a candidate token outside [0, V), more trie nodes than
 *   R (UNO_DEV_BAD_DRAFT) or a NaN logit in a row the walk reads
 *   (UNO_DEV_NAN) set the status bits; that sequence's outputs are -1.
 *   workspace: >= uno_tree_verify_workspace(B, N, k, R, V) bytes, 16-byte
 *   aligned, any contents.
 * ------------------------------------------------------------------------- */
size_t uno_tree_verify_workspace(int32_t B, int32_t N, int32_t k, int32_t R, int32_t V);

uno_status uno_tree_verify(uno_dtype dt, int32_t B, int32_t N, int32_t k, int32_t R, int32_t V,
                           const void* p_logits, const void* q_logits, const int32_t* cands,
                           int32_t bonus, float temperature, uint64_t seed, uint64_t step,
                           uint64_t seq_offset, int32_t* accepted_len, int32_t* out_tokens,
                           int32_t* out_count, int32_t* dev_status, void* workspace,
                           size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Distillation losses (hyper.ai page, section "方法": the adapter is trained
 * with alpha * L_DCD + beta * L_TV on one gated forward pass, the clean rows
 * (gate 0) giving the teacher logits, the noisy rows (gate 1) the student's):
 *   per row i: p = softmax(z_teacher[i] / T), q = softmax(z_student[i] / T),
 *     losses[i] = (KL(p || q), TV(p, q) = 1/2 sum |p - q|);
 *   grad[i] (optional) = d(alpha * mean KL + beta * mean TV) / d z_student[i]
 *     = (alpha (q - p) + beta q (s - sum_v s_v q_v) / 2) / (T rows),
 *     s = sign(q - p) (0 where p = q).
 *   z_teacher, z_student [rows, V] `dt`, 16-byte aligned; losses [rows, 2]
 *   float; grad [rows, V] float or NULL (losses only). No workspace.
 *   A NaN logit in a row pair: that pair's losses (and gradient) are NaN and
 *   UNO_DEV_NAN is set in dev_status (may be NULL).
 * ------------------------------------------------------------------------- */
uno_status uno_distill(uno_dtype dt, int32_t rows, int32_t V, const void* z_teacher,
                       const void* z_student, float alpha, float beta, float temperature,
                       float* losses, float* grad, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Verification and draft with the vocabulary split over G devices (the LM
 * head's rows sharded; hyper.ai page, section "方法", the Psi-Spec
 * paragraph: the test against the AR distribution needs its normaliser over
 * the whole vocabulary, the residual and bonus draws cumulative mass in
 * vocabulary order). Device `rank` holds the logits of its contiguous shard
 * [v0, v0 + Vs) of the V ids, shards in rank order. Per step, on every device:
 *   1. uno_vp_partials on its AR rows (id_kind 1) and draft rows (id_kind 2):
 *      out [rows, 4] float = (m, s, z(d), 0) with m the row max over the
 *      shard, s = sum 2^((z - m) log2(e) / T), z(d) the drafted token's logit
 *      when the shard holds it (else -inf);
 *   2. all-gather them ([G, rows, 4], rank order), then uno_vp_verify_decide:
 *      the merged normalisers give p(d), q(d) and the same acceptance, first
 *      rejection n and outputs as uno_psi_verify on every device, except the
 *      drawn token: out_tokens[b, pos] = -1 at the draw position pos = draw[b]
 *      (n < k residual, k bonus, -1 no draw); draw_stats [B, 4] float holds the
 *      merged (Mp, Sp, Mq, Sq) of the draw row;
 *   3. uno_vp_draw_masses: masses [B, 2] double = the draw row's residual mass
 *      sum max(p - q, 0) (the bonus: p mass) and p mass over the shard;
 *   4. all-gather them ([G, B, 2]), then uno_vp_draw: the shard holding
 *      u * Z in rank order (u as in uno_psi_verify; a zero residual mass
 *      falls back to p) writes the drawn global id at out_tokens[b, pos];
 *      the others leave -1;
 *   5. an all-reduce MAX of out_tokens over the devices gives every device
 *      the tokens uno_psi_verify would emit.
 * The next block's draft: uno_vp_partials on the shard's draft-logit rows
 * (id_kind 0, precise 1: the float-pair scale of the single-device draft),
 * all-gather, uno_vp_draft_draw (the owner writes the global id, the others
 * -1), all-reduce MAX. Results equal the single-device calls up to the order
 * of floating-point sums. Logits `dt`, 16-byte aligned rows (Vs a multiple of
 * 8 for bf16); partial and mass buffers 16-byte aligned; 1 <= G <= 64.
 * ------------------------------------------------------------------------- */
uno_status uno_vp_partials(uno_dtype dt, int32_t rows, int32_t Vs, int32_t v0, const void* logits,
                           const int32_t* draft, int32_t k, int32_t k_p, int32_t id_kind,
                           int32_t precise, float temperature, float* out, void* stream);

uno_status uno_vp_verify_decide(int32_t B, int32_t k, int32_t k_p, int32_t V, int32_t G,
                                const float* parts_p, const float* parts_q, const int32_t* draft,
                                float temperature, uint64_t seed, uint64_t step,
                                uint64_t seq_offset, int32_t* accepted_len, int32_t* out_tokens,
                                int32_t* out_count, int32_t* draw, float* draw_stats,
                                int32_t* dev_status, void* stream);

uno_status uno_vp_draw_masses(uno_dtype dt, int32_t B, int32_t k, int32_t k_p, int32_t Vs,
                              const void* p_shard, const void* q_shard, const int32_t* draw,
                              const float* draw_stats, float temperature, double* masses,
                              void* stream);

uno_status uno_vp_draw(uno_dtype dt, int32_t B, int32_t k, int32_t k_p, int32_t Vs, int32_t v0,
                       int32_t V, int32_t G, int32_t rank, const void* p_shard,
                       const void* q_shard, const int32_t* draw, const float* draw_stats,
                       const double* masses_all, float temperature, uint64_t seed, uint64_t step,
                       uint64_t seq_offset, int32_t* out_tokens, void* stream);

uno_status uno_vp_draft_draw(uno_dtype dt, int32_t B, int32_t k, int32_t Vs, int32_t v0, int32_t V,
                             int32_t G, int32_t rank, const void* q_shard, const float* parts_all,
                             float temperature, uint64_t seed, uint64_t step, uint64_t seq_offset,
                             int32_t* draft, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Linear-sampler draft (hyper.ai page, section "方法": the linear sampler
 * draws one candidate block from the per-position marginals):
 *   draft[b,j] = smallest v with C(v) > u0 * C(V-1), C the inclusive
 *   cumulative sum of softmax(q_logits[b,j] / T) in ascending id; u0 from
 *   Philox stream 0 at index (seq_offset + b)*k + j.
 *   q_logits [B,k,V] `dt`; draft [B,k] int32 (device).
 *   workspace: >= uno_draft_sample_workspace(B, k, V) bytes, 16-byte
 *   aligned, any contents (per-row, per-vocab-chunk softmax statistics).
 *   A row holding a NaN logit gets draft -1 and sets UNO_DEV_NAN.
 * ------------------------------------------------------------------------- */
size_t uno_draft_sample_workspace(int32_t B, int32_t k, int32_t V);

uno_status uno_draft_sample(uno_dtype dt, int32_t B, int32_t k, int32_t V, const void* q_logits,
                            float temperature, uint64_t seed, uint64_t step, uint64_t seq_offset,
                            int32_t* draft, int32_t* dev_status, void* workspace,
                            size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Philox uniforms, exposed so the generator can be checked bit for bit:
 *   words[i] = Philox4x32-10 word 0 at counter (index0 + i, step lo, step hi,
 *   stream), key (seed lo, seed hi); u[i] = (words[i] >> 8) * 2^-24.
 *   Either output may be NULL. n >= 0, index0 + n <= 2^32.
 * ------------------------------------------------------------------------- */
uno_status uno_philox_uniforms(uint64_t seed, uint64_t step, uint32_t stream_id, uint32_t index0,
                               int64_t n, uint32_t* words, float* u, void* stream);

/* ---------------------------------------------------------------------------
 * Synthetic decode step (the linear decode step of Psi-Spec on a stand-in
 * decoder stack: gated-LoRA projections of every layer, no attention; the
 * model-side rules come from hyper.ai page, section "方法", the shapes from
 * section "实验" — rank-128 adapters on Qwen3-8B):
 *
 *   per layer:  n = rmsnorm(h); q = L_q(n); k = L_k(n); v = L_v(n) (unused);
 *               h = h + L_o(q); n = rmsnorm(h);
 *               h = h + L_down(silu(L_gate(n)) * L_up(n))
 *   logits = L_head(rmsnorm(h)), rmsnorm(x) = x / sqrt(mean(x^2) + 1e-6)
 *
 * with L = the gated-LoRA linear above, bf16 storage between operations.
 *
 * Model handle: holds device pointers and cached launch descriptors only;
 * the caller owns (and keeps alive) the weight memory. `weights` lists, for
 * each layer in order, the (W, A, Bl) device pointers of q, k, v, o, gate, up,
 * down (21 per layer), then those of the LM head: 21 * n_layers + 3 pointers.
 * Shapes: q [q_out, hidden], k and v [kv_out, hidden], o [hidden, q_out],
 * gate and up [inter, hidden], down [hidden, inter], head [vocab, hidden];
 * A [r, in], Bl [out, r]. All bf16.
 * ------------------------------------------------------------------------- */
typedef struct uno_model uno_model;

uno_status uno_model_create(uno_model** out, int32_t n_layers, int32_t hidden, int32_t q_out,
                            int32_t kv_out, int32_t inter, int32_t vocab, int32_t r, float scale,
                            const void* const* weights);
void uno_model_destroy(uno_model* m);

/* One step for B sequences with block size k (M = B(2k+1) rows):
 *   h_in [M, hidden] bf16: rows 0..B(k+1)-1 are the verify rows (gate 0,
 *     sequence-major: anchor + k drafted tokens), then B*k mask rows
 *     (gate 1) that produce the next block's draft distributions.
 *   Verifies the previous block (q_prev [B,k,V] bf16, d_prev [B,k] int32)
 *   against this step's AR rows p [B,k+1,V] (bonus enabled), as
 *   uno_psi_verify with k_p = k+1 and the same seed/step/seq_offset (global
 *   sequence ids seq_offset + b: a batch split over ranks draws what the
 *   whole batch would); then drafts the next block from the mask rows as
 *   uno_draft_sample (same seed/step/seq_offset) into
 *   d_next [B,k], and writes their logits to q_next [B,k,V] bf16.
 *   logits_out: optional [B(k+1), V] bf16 copy target for the AR rows (NULL
 *   to skip). accepted_len [B], out_tokens [B,k+1], out_count [B] as in
 *   uno_psi_verify. q_next must not alias q_prev.
 *   workspace: >= uno_psi_step_workspace(m, B, k) bytes, 16-byte aligned,
 *   any contents (the step clears the stream-K flags it holds on `stream`
 *   first). Steps that share a workspace must not run at the same time. */
size_t uno_psi_step_workspace(const uno_model* m, int32_t B, int32_t k);

uno_status uno_psi_step(uno_model* m, int32_t B, int32_t k, const void* h_in, const void* q_prev,
                        const int32_t* d_prev, float temperature, uint64_t seed, uint64_t step,
                        uint64_t seq_offset, void* q_next, int32_t* d_next, void* logits_out,
                        int32_t* accepted_len, int32_t* out_tokens, int32_t* out_count,
                        int32_t* dev_status, void* workspace, size_t ws_bytes, void* stream);

/* The decoder-layer part of uno_psi_step, for inspecting a step layer by
 * layer. Each layer has two residual sub-blocks: 2l (rmsnorm, q/k/v, h += o(q))
 * and 2l+1 (rmsnorm, h += down(silu(gate) * up)). This call runs the launches
 * uno_psi_step issues for the first n_blocks sub-blocks (0 <= n_blocks <=
 * 2 * layers; the same kernels, launch shapes and workspace layout as a step
 * with this B and k) on h_in [M, hidden] bf16, M = B(2k+1), and writes the
 * hidden state after them to h_out [M, hidden] (h_out may alias h_in).
 * Optional outputs (NULL to skip), all [M, width] bf16: q_out [M, q_out],
 * k_out and v_out [M, kv_out] of the last projection sub-block run
 * (n_blocks >= 1), act_out = silu(gate) * up [M, inter] of the last MLP
 * sub-block run (n_blocks >= 2). workspace: as for uno_psi_step. No LM head,
 * verify or draft. */
uno_status uno_psi_step_hidden(uno_model* m, int32_t B, int32_t k, const void* h_in,
                               int32_t n_blocks, void* h_out, void* q_out, void* k_out,
                               void* v_out, void* act_out, void* workspace, size_t ws_bytes,
                               void* stream);

/* Number of kernel launches one uno_psi_step call with this (B, k) issues;
 * 0 until such a step has been run (the launch plan is built on first use). */
int32_t uno_psi_step_kernel_count(const uno_model* m, int32_t B, int32_t k);

/* Launch timing of uno_psi_step (a library addition for measurement; the
 * pages have no counterpart). With enable != 0, every later uno_psi_step on
 * this model records a CUDA event on its stream before its first launch and
 * after each launch of its plan, after the verification's two kernels and
 * after the draft's two; uno_model_last_profile then waits for the last
 * profiled step and reports, per entry i in launch order:
 *   ms[i]    the time between the event before and the event after it (the
 *            time the entry adds to the stream; the events themselves can
 *            cost some of the overlap between consecutive launches);
 *   kind[i]  0 one-CTA GEMM, 1 CTA-pair GEMM, 2 CTA-pair GEMM that computes
 *            the LoRA activations t itself, 3 fused decode-size GEMM,
 *            10 RMSNorm, 11 RMSNorm + LoRA down-projection, 12 rows' sums
 *            of squares (steps of 512 rows and more fold RMSNorm into
 *            their GEMMs and launch this once for the input),
 *            20 verification (stats + finalize), 21 draft (stats + draw);
 *   dims[4i .. 4i+3] (optional, may be NULL) for GEMMs: M, the summed N of
 *            its output groups, K and the epilogue mode (0 store, 1 residual
 *            add, 2 gated down-projection, 3 silu pair); zeros otherwise.
 * *n_out receives the number of entries (0 before a profiled step); with
 * ms == NULL nothing else is written (a count query); otherwise cap is the
 * length of ms and kind (dims: 4 cap) and must hold every entry. Events are created on the device
 * of the first profiled step; profiled steps and the read must use that
 * device (UNO_ERR_INVALID_ARG otherwise). enable = 0 stops recording. */
uno_status uno_model_profile(uno_model* m, int32_t enable);
uno_status uno_model_last_profile(uno_model* m, int32_t cap, float* ms, int32_t* kind,
                                  int64_t* dims, int32_t* n_out);

/* ---------------------------------------------------------------------------
 * Self-test of the bounded waits (a library addition; the pages have no
 * counterpart). Every spin in the library's kernels gives up after a time
 * limit, ORs UNO_DEV_TIMEOUT into the status words and returns, so a lost
 * arrival ends in a status the host reads, never in a hung GPU. This call
 * runs one such wait on a condition nothing will satisfy, with no copy or
 * tensor-core work in flight:
 *   which 0: a global-memory flag that is never raised;
 *         1: an mbarrier phase that gets no arrival;
 *         2: the same through the cluster-scope wait (used between CTA pairs);
 *         3: control: the expected arrival comes first and the wait succeeds.
 *   limit_ns in [1e3, 1e8]; result: device int32, 1 if the wait was
 *   satisfied, 0 if it gave up; dev_status: optional device int32 word.
 * ------------------------------------------------------------------------- */
uno_status uno_wait_selftest(int32_t which, uint64_t limit_ns, int32_t* result,
                             int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * The step's glue operations, exposed for testing (all bf16, device):
 *   uno_rmsnorm:  y[m,:] = x[m,:] / sqrt(mean(x[m,:]^2) + eps)      x, y [M,D]
 *   uno_silu_mul: y = silu(a) * b = a / (1 + exp(-a)) * b           [n]
 * ------------------------------------------------------------------------- */
uno_status uno_rmsnorm(int64_t M, int64_t D, const void* x, void* y, float eps, void* stream);
uno_status uno_silu_mul(int64_t n, const void* a, const void* b, void* y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* UNO_H_ */
