/*
 * sla.h -- C ABI of the B200 (sm_100a) SLA / SLA2 sparse-linear attention.
 *
 * One call, sla_forward(), runs the whole forward of a batch of heads on one
 * GPU, every step in this library's CUDA kernels:
 *
 *   1. block mean pooling of Q and K over 64-token blocks (SLA2: followed by the
 *      learnable router projections proj_q / proj_k);
 *   2. pooled scores s_ij = qbar_i . kbar_j and the per-row three-way block
 *      classification into the compressed mask Mc (1 critical, 0 marginal,
 *      -1 negligible) plus the ascending index lists of critical / negligible
 *      blocks;
 *   3. phi(K) (softmax over the head dimension) and the linear-attention sums
 *      h_j = phi(K_j)^T V_j, z_j = rowsum(phi(K_j)^T);
 *   4. per 64-row query block: softmax attention over the critical key blocks
 *      (online softmax, tensor cores), the linear branch
 *      phi(Q_i) H_i / phi(Q_i) Z_i over the marginal blocks, and the combine
 *      (SLA: O = O^s + O^l W; SLA2: O = alpha_h O^s + (1 - alpha_h) O^l).
 *
 * Beside it: sla_dense_forward() (the dense baseline), sla_router_soft_topk()
 * (SLA2's differentiable router for its first training stage),
 * sla_forward_train() and sla_backward() (the gradients of the forward), and
 * read-back and timing helpers.
 *
 * Sources (page title, section):
 *   - "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
 *     Sparse-Linear Attention", structured summary (aipaper.cc), section 4
 *     "Methodology": formula 1 (Pc from pooled Q, K), formula 2 (Mc), formula 3
 *     (H_i, Z_i, O^l_i), formula 4 (O = O^s + Proj(O^l)).
 *   - SLA walkthrough (intelliparadigm.com), sections 1.2 and 2.2: bq = bkv = 64,
 *     precomputed h_j / z_j, online softmax, one fused kernel; section 3.2:
 *     phi = softmax.
 *   - SLA2 article, arXiv 2602.12675 (mcffsbgs.com): O = alpha O^s +
 *     (1 - alpha) O^l, router with two projection matrices, low-bit Q, K, P, V.
 *   - "SLA2 -- L3 Cross-Paper Synthesis" (zhaifeiyue.github.io), section 2:
 *     alpha mixing replaces SLA's projection; router proj_q / proj_k.
 *
 * Conventions
 *   - Q, K, V, O: contiguous row-major [B, H, N_pad, d] bfloat16 in device
 *     memory, N_pad = 64 * ceil(N / 64). Rows N .. N_pad-1 of Q, K, V are pad:
 *     never read into any result (they may hold anything, NaN included).
 *     Rows N .. N_pad-1 of O are not written. Base addresses 16-byte aligned.
 *   - d is 64 or 128. Block sizes are fixed at 64 x 64.
 *   - Every call is asynchronous on the given stream (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream) and enqueues only kernels,
 *     cudaMemsetAsync and cudaMemcpyAsync. The library never allocates or frees
 *     memory and never synchronises, except sla_read_device_status().
 *   - Ownership: the caller owns every buffer (inputs, outputs, weights and the
 *     workspace) and must keep them alive until the stream work completes.
 *   - Errors are returned as sla_status codes; arguments are validated before
 *     anything is enqueued, so a non-SLA_OK return from validation means
 *     nothing ran. SLA_ERR_CUDA reports a launch or runtime error.
 *   - Reentrancy: calls may run concurrently on different streams if each uses
 *     its own workspace. Results are deterministic: the same inputs give
 *     bitwise identical O, Mc and index lists (no floating-point atomics).
 */
#ifndef SLA_H_
#define SLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SLA_ABI_VERSION 5 /* 2: sla_params.phi; 3: sla_router_soft_topk; 4: training forward, backward;
                             5: sla_forward_noalloc, sla_read_device_status(NULL), sla_check_wait_timeout */
#define SLA_BLOCK 64
#define SLA_MAX_BLOCKS 4096 /* N <= 262144 */

typedef enum {
  SLA_OK = 0,
  SLA_ERR_INVALID_ARG = 1,    /* a null pointer, a bad size or count, a bad enum value */
  SLA_ERR_UNSUPPORTED = 2,    /* valid request this build does not implement (e.g. d not 64/128) */
  SLA_ERR_WORKSPACE = 3,      /* workspace missing, misaligned (256 B) or smaller than required */
  SLA_ERR_ALIGNMENT = 4,      /* a tensor base address not 16-byte aligned */
  SLA_ERR_CUDA = 5,           /* a CUDA launch or runtime call failed */
  SLA_ERR_DEVICE_TIMEOUT = 6, /* a bounded wait inside a kernel expired (see sla_read_device_status) */
  SLA_ERR_DEVICE_CHECK = 7    /* an in-kernel consistency check failed (e.g. a block index out of range) */
} sla_status;

typedef enum { SLA_VARIANT_SLA = 0, SLA_VARIANT_SLA2 = 1 } sla_variant;

typedef enum {
  SLA_PREC_BF16 = 0,      /* bf16 tensor-core products, fp32 accumulation */
  SLA_PREC_I8QK_F8PV = 1  /* sparse branch with INT8 Q K^T and FP8 e4m3 P V */
} sla_precision;

/* Feature map phi of the linear branch, applied to every query and key row.
 * SLA structured summary, section 4: phi is an activation such as softmax or
 * ELU+1 (its Table 2 ablates both); the SLA walkthrough (section 3.2) and the
 * SLA2 notes choose softmax. */
typedef enum {
  SLA_PHI_SOFTMAX = 0, /* softmax over the head dimension, max-subtracted */
  SLA_PHI_ELU1 = 1     /* elu(x) + 1 elementwise: x + 1 for x > 0, exp(x) otherwise */
} sla_phi;

typedef struct sla_params {
  int B, H;            /* batch and heads (>= 1) */
  int N;               /* true sequence length (>= 1); tensors hold N_pad rows */
  int d;               /* head dimension: 64 or 128 */
  int block_q;         /* must be 64 */
  int block_kv;        /* must be 64 */
  int variant;         /* sla_variant */
  int precision;       /* sla_precision */
  int k_crit;          /* critical blocks per row: 1 <= k_crit <= Nb */
  int k_neg;           /* negligible blocks per row: 0 <= k_neg, k_crit + k_neg <= Nb */
  float softmax_scale; /* scale of q.k in the sparse branch; 0 selects 1/sqrt(d) */
  const void* w_proj;  /* SLA: [d, d] bf16 device, y = x W (row-major [in][out]); NULL = identity */
  const void* proj_q;  /* SLA2 router: [d, d] bf16 device, qbar W_q; NULL = none (both or neither) */
  const void* proj_k;  /* SLA2 router: [d, d] bf16 device, kbar W_k */
  const float* alpha;  /* SLA2: [H] float32 device, per-head mixing weight; required for SLA2 */
  int phi;             /* sla_phi; 0 (softmax) for the method as published */
} sla_params;

/* ABI version of the loaded library (SLA_ABI_VERSION at build time). */
int sla_abi_version(void);

/* Static description of a status code; never NULL. */
const char* sla_status_string(sla_status status);

/* Bytes of device workspace sla_forward() needs for these parameters, or 0 if
 * the parameters are invalid (call sla_validate for the reason). */
size_t sla_workspace_size(const sla_params* p);

/* Checks the parameters alone (no pointers to tensors): SLA_OK or the error
 * sla_forward would return for them. */
sla_status sla_validate(const sla_params* p);

/* The forward pass (steps 1-4 above).
 *   Q, K, V   [B, H, N_pad, d] bf16 device inputs.
 *   O         [B, H, N_pad, d] bf16 device output (rows >= N untouched).
 *   workspace device scratch of at least sla_workspace_size(p) bytes,
 *             256-byte aligned; its contents on entry do not matter. After the
 *             call it holds the pooled vectors, Mc and the index lists
 *             (read them with sla_get_mask / sla_get_pooled) until reused.
 *   stream    cudaStream_t as void*. */
sla_status sla_forward(const void* Q, const void* K, const void* V, void* O, const sla_params* p,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Training: the backward pass.
 * Source: SLA walkthrough (intelliparadigm.com), section 2.3: the sparse path
 * takes the FlashAttention backward on the Mc = 1 blocks, the linear path the
 * gradients of phi(Q), phi(K) and V by the chain rule, block by block.
 *
 * Activations a training forward keeps for sla_backward (device buffers owned
 * by the caller; rows N .. N_pad-1 are not written). */
typedef struct sla_saved {
  void* o_s;   /* [B, H, N_pad, d] bf16: the sparse branch O^s */
  void* o_l;   /* [B, H, N_pad, d] bf16: the linear branch O^l (SLA: before W) */
  float* lse;  /* [B, H, N_pad] float32: log sum_t exp(scale q.k_t) over the row's critical keys */
  float* den;  /* [B, H, N_pad] float32: phi(q) . Z_i, 0 where the row has no marginal block */
} sla_saved;

/* sla_forward (same arguments and result) that also writes the activations of
 * `saved` (every pointer required, 16-byte aligned bf16 / 4-byte float32).
 * bf16 precision only (SLA_ERR_UNSUPPORTED otherwise). Keep the workspace and
 * `saved` unchanged until sla_backward has run on them. */
sla_status sla_forward_train(const void* Q, const void* K, const void* V, void* O, const sla_params* p,
                             const sla_saved* saved, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace sla_backward() needs (0 for invalid parameters). */
size_t sla_backward_workspace_size(const sla_params* p);

/* Gradients of <dO, O> for the forward of sla_forward_train with the block
 * mask held fixed (a hard Top-k has no gradient; no gradient reaches the
 * router projections or the pooling).
 *   Q, K, V, dO   [B, H, N_pad, d] bf16 device inputs; rows >= N of dO are ignored.
 *   p, saved      the parameters and activations of the training forward.
 *   fwd_workspace its workspace (mask, block lists, phi(K), z_j, H_tot, Z_tot).
 *   dQ, dK, dV    [B, H, N_pad, d] bf16 device outputs; rows >= N are written as 0.
 *   dW            SLA: [d, d] float32 device output, sum over batch and heads of
 *                 O^l^T dO (the gradient of W); may be NULL. Must be NULL for SLA2.
 *   dalpha        SLA2: [H] float32 device output, sum over the batch of
 *                 dO . (O^s - O^l); may be NULL. Must be NULL for SLA.
 *   workspace     at least sla_backward_workspace_size(p) bytes, 256-byte aligned.
 * bf16 precision only. The result is deterministic (no floating-point atomics).
 * A bounded in-kernel wait that expires during the backward is recorded in
 * the forward workspace's status word: check it with
 * sla_read_device_status(fwd_workspace, stream). */
sla_status sla_backward(const void* Q, const void* K, const void* V, const void* dO, const sla_params* p,
                        const sla_saved* saved, const void* fwd_workspace, size_t fwd_workspace_bytes, void* dQ,
                        void* dK, void* dV, float* dW, float* dalpha, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Copies the compressed mask and block lists of the last sla_forward() that
 * used this workspace (stream-ordered, device to device; any output may be NULL).
 *   mc    [B, H, Nb, Nb] int8: 1 critical, 0 marginal, -1 negligible.
 *   crit  [B, H, Nb, k_crit] int32, ascending block indices.
 *   neg   [B, H, Nb, k_neg] int32, ascending block indices. */
sla_status sla_get_mask(const sla_params* p, const void* workspace, int8_t* mc, int32_t* crit,
                        int32_t* neg, void* stream);

/* Copies the pooled (SLA2: pooled and router-projected) vectors the mask was
 * ranked on, [B, H, Nb, d] float32 each (device to device; either may be NULL). */
sla_status sla_get_pooled(const sla_params* p, const void* workspace, float* qbar, float* kbar,
                          void* stream);

/* Quantised sparse branch (precision SLA_PREC_I8QK_F8PV): copies the codes and
 * per-block scales of the last sla_forward() on this workspace (device to
 * device; any output may be NULL). Source: SLA2 article (mcffsbgs.com),
 * quantisation paragraphs (Q, K, P, V to low-bit values with scaling).
 *   qcode, kcode  [B, H, N_pad, d] int8: clamp(rint(x / s), -127, 127), rows >= N zero.
 *   vcode         [B, H, N_pad, d] FP8 e4m3 bytes: e4m3(v / s), RNE, saturating.
 *   qscale, kscale [B, H, Nb] float32: absmax / 127 over the block's valid rows (1 if 0).
 *   vscale        [B, H, Nb] float32: absmax / 448 (1 if 0).
 * Returns SLA_ERR_INVALID_ARG for a bf16-precision parameter set. */
sla_status sla_get_quantized(const sla_params* p, const void* workspace, int8_t* qcode, int8_t* kcode,
                             uint8_t* vcode, float* qscale, float* kscale, float* vscale, void* stream);

/* SoftTop-k router forward, the differentiable stand-in for the hard Top-k in
 * the first training stage of SLA2's router. Sources: SLA2 article
 * (mcffsbgs.com), two-stage training paragraphs (a sigmoid with a temperature
 * replaces Top-k); "SLA2 -- L3 Cross-Paper Synthesis" (zhaifeiyue.github.io),
 * section 3 (lambda_i per row by binary search on the row-sum constraint);
 * SLA structured summary (aipaper.cc), section 4, formula 1 (Pc).
 *
 * Runs step 1 of sla_forward (pooling; SLA2 with proj_q / proj_k: the router
 * projections) and the pooled scores s_ij, then per row i:
 *   Pc_ij = softmax_j(scale s_ij), scale = p->softmax_scale or 1/sqrt(d);
 *   M_ij  = sigmoid((Pc_ij - lambda_i) / tau), lambda_i the unique root of
 *           sum_j M_ij = k_crit, found in float32 inside a shrinking bracket
 *           (Newton steps, bisection where a step would leave the bracket).
 * k_crit = Nb gives M = 1 and lambda = -inf. p->k_neg, w_proj, alpha and phi
 * are not used (p must still validate as for sla_forward).
 *   Q, K      [B, H, N_pad, d] bf16 device inputs (as sla_forward).
 *   tau       temperature: finite, > 0, and 1/tau finite.
 *   m_soft    [B, H, Nb, Nb] float32 device output (required).
 *   lambda    [B, H, Nb] float32 device output, or NULL.
 *   pc        [B, H, Nb, Nb] float32 device output, or NULL.
 *   workspace at least sla_workspace_size(p) bytes, 256-byte aligned; it
 *             holds the pooled vectors and scores afterwards (sla_get_pooled).
 * Errors: SLA_ERR_INVALID_ARG for a bad tau or a null Q, K or m_soft;
 * otherwise as sla_forward. */
sla_status sla_router_soft_topk(const void* Q, const void* K, const sla_params* p, float tau,
                                float* m_soft, float* lambda, float* pc, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Synchronises the stream, then reads the device status word written by the
 * last sla_forward() on this workspace: SLA_OK, SLA_ERR_DEVICE_TIMEOUT if a
 * bounded in-kernel wait gave up, or SLA_ERR_DEVICE_CHECK if an in-kernel check
 * failed (in both cases the output is not valid). workspace = NULL reads the
 * status word of the last sla_forward_noalloc() on the current device. */
sla_status sla_read_device_status(const void* workspace, void* stream);

/* Failure-detection self-test (no counterpart on the pages). Every wait of the
 * library's kernels on an mbarrier is bounded: when it expires, the kernel
 * writes SLA_ERR_DEVICE_TIMEOUT's code into the workspace's status word and
 * returns instead of hanging. This call makes exactly that happen, harmlessly:
 * one thread waits, with the same wait routine, on an mbarrier that nothing
 * arrives on, giving up after limit_cycles SM cycles (1 .. 4e9; the forward's
 * kernels use 4e9, about 2 s). Nothing else is in flight, so the kernel returns
 * normally and the context stays usable. Afterwards sla_read_device_status()
 * on the same workspace returns SLA_ERR_DEVICE_TIMEOUT; the next sla_forward()
 * on it clears the word.
 *   workspace  device buffer of at least 256 bytes, 256-byte aligned (a forward
 *              workspace may be used; only its status word is touched).
 * Errors: SLA_ERR_WORKSPACE, SLA_ERR_INVALID_ARG for a limit out of range. */
sla_status sla_check_wait_timeout(void* workspace, size_t workspace_bytes, long long limit_cycles,
                                  void* stream);

/* Dense softmax attention O = softmax(Q K^T * scale) V over all N keys, with
 * the same kernel machinery as the sparse branch (every block critical, no
 * linear branch, no mask). The baseline the pages compare against
 * (FlashAttention, SLA structured summary section 6, kernel-speed figure).
 * Same tensor layout as sla_forward; no workspace. */
sla_status sla_dense_forward(const void* Q, const void* K, const void* V, void* O, int B, int H,
                             int N, int d, float softmax_scale, void* stream);

/* Forward pass for callers that cannot allocate device memory (no counterpart
 * on the pages: it is a deployment aid). Some host programs own all GPU memory
 * themselves (a plugin inside a server or engine with a fixed memory pool, a
 * statically planned embedded deployment) or must not call cudaMalloc while
 * running, since it can synchronise the device. They pass Q, K, V, O and the
 * parameters exactly as for sla_forward, but no workspace.
 *
 * The scratch comes from one static device array of SLA_NOALLOC_WORKSPACE_BYTES
 * (32 MiB) inside the library, held by every GPU that loads the library until
 * the process exits. The call allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine).
 *   - Returns SLA_ERR_WORKSPACE, before enqueueing anything, when
 *     sla_workspace_size(p) exceeds SLA_NOALLOC_WORKSPACE_BYTES.
 *   - The first call on a device looks up the array's device address for that
 *     device (cudaGetSymbolAddress, with that device current); make that first
 *     call before any stream capture begins.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; each call re-initialises what must start at zero. Calls whose
 *     GPU work overlaps (different streams, different host threads without
 *     ordering) race on the array and give undefined results: order them on
 *     one stream or serialise them.
 *   - The mask and lists of these calls live in the shared array and are not
 *     readable through sla_get_mask. Their device status word is: pass NULL as
 *     the workspace of sla_read_device_status. A bounded in-kernel wait that
 *     expires in a no-alloc call (SLA_ERR_DEVICE_TIMEOUT, output not valid) is
 *     reported only there: the call itself has already returned SLA_OK. */
#define SLA_NOALLOC_WORKSPACE_BYTES (32u << 20)
sla_status sla_forward_noalloc(const void* Q, const void* K, const void* V, void* O,
                               const sla_params* p, void* stream);

/* Stage timing, a profiling aid (no counterpart on the pages). Stages of
 * sla_forward, in order: 0 the Q-side pass (pooling of Q, + router; phi(Q) when
 * the linear branch takes it precomputed; at d = 64 or with the quantised
 * branch also the pooling of K and the INT8 codes), 1 the K / V pass (at d = 128
 * in bf16 also the pooling of K; phi(K), z_j, partial H and Z), 2 pooled
 * scores, 3 classification, 4 H_tot / Z_tot reduction (and Z_i), 5 attention
 * (sparse + linear + combine). */
#define SLA_NUM_STAGES 6

/* max_calls > 0: create CUDA events (on the current device) for up to max_calls
 * sla_forward calls and start recording: each call records an event before its
 * first stage and after every stage, on its stream. 0: stop and release the
 * events. Process-wide state, not thread-safe; off by default. */
sla_status sla_stage_timing(int max_calls);

/* Waits for the recorded events, writes the summed elapsed milliseconds of each
 * stage over the recorded calls to ms[SLA_NUM_STAGES] and their number to
 * *calls, then clears the record (recording continues). */
sla_status sla_stage_times(float* ms, int* calls);

#ifdef __cplusplus
}
#endif

#endif /* SLA_H_ */
