/*
 * la_api.h — C ABI of the B200 kernelized linear-attention library
 * (liblinattn.so).
 *
 * The operation (per batch b and head h; tensors [B, H, N, D], D innermost):
 *
 *     a_i = phi(q_i),   b_j = phi(k_j)
 *     S_i = sum_{j in J(i)} b_j v_j^T   (D x D),   z_i = sum_{j in J(i)} b_j
 *     o_i = S_i^T a_i / (a_i . z_i)
 *
 * J(i) is every key (non-causal) or j <= i (causal).  This is the
 * kernel-decomposition form of attention in "Efficient Transformers Survey",
 * section Linear Attention, Proposition "Linear Attention via Kernel
 * Decomposition" (Statement: S and z are precomputed sums, each output is one
 * query against them); the causal prefix and the decode step are the
 * recurrent computation of the same proposition ("Why It Matters": S and z
 * updated token by token, constant memory per step).  The backward pass
 * ("Transformer Based Linear Attention with Optimized GPU Kernel
 * Implementation", Abstract: forward and backward passes of O(N D^2) cost)
 * returns the gradients of sum(dO * O) with respect to q, k and v.
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers, contiguous [B, H, N, D] (or
 *     [B, H, D] for decode vectors, [B, H, D, D] for states), 16-byte
 *     aligned.  Element type: `dt` for q, k, v, o, dO, dq, dk, dv; float32
 *     always for states (S, z) and the workspace.
 *   - The caller owns all memory.  The library never allocates or frees
 *     device memory.  Calls that need scratch take a caller-provided
 *     workspace of at least la_workspace_size() bytes (256-byte aligned).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and never synchronises the host.
 *   - Arguments are validated before anything is launched.  Invalid input
 *     returns a status; nothing crosses the ABI as an exception or abort.
 *   - phi is LA_PHI_ELU1: elu(x)+1 (= x+1 for x > 0, exp(x) otherwise) or
 *     LA_PHI_RELU_EPS: max(x, 0) + 1e-6.  Both are > 0, so no epsilon is
 *     added to the denominator.  LA_PHI_IDENTITY takes q and k as feature
 *     vectors already (the caller keeps them positive).
 *   - Supported head sizes D: 16, 32, 64, 128.  N, B, H >= 0 (a zero size
 *     launches nothing and returns LA_OK; a requested final state is then
 *     zero-filled).  B*H*N*D must stay below 2^62, N below 2^31.
 *   - Accumulation is float32 throughout; bf16 inputs are read exactly.
 */
#ifndef LA_API_H
#define LA_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LA_API_VERSION 2

#if defined(__GNUC__)
#define LA_EXPORT __attribute__((visibility("default")))
#else
#define LA_EXPORT
#endif

/* ABI-identical to cudaStream_t; declared here so this header needs no CUDA
 * headers. */
typedef struct CUstream_st *la_stream_t;

typedef enum la_status {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, negative size, bad enum */
    LA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. D = 48) */
    LA_ERR_CUDA = 3,           /* a CUDA launch or runtime call failed */
    LA_ERR_WORKSPACE = 4,      /* workspace missing or smaller than required */
    LA_ERR_DEVICE_TIMEOUT = 5  /* a bounded on-device wait gave up (see below) */
} la_status;

typedef enum la_phi {
    LA_PHI_ELU1 = 0,      /* elu(x) + 1 */
    LA_PHI_RELU_EPS = 1,  /* max(x, 0) + 1e-6 */
    LA_PHI_IDENTITY = 2   /* q, k are feature vectors already (positive: e.g. the
                             output of la_favor_features); phi' = 1, so the
                             backward returns the features' gradients */
} la_phi;

typedef enum la_dtype {
    LA_F32 = 0,   /* float32 tensors */
    LA_BF16 = 1   /* bfloat16 tensors, float32 accumulation */
} la_dtype;

typedef enum la_op {
    LA_OP_FORWARD = 0,
    LA_OP_BACKWARD = 1
} la_op;

/*
 * Bytes of device workspace that la_forward (op = LA_OP_FORWARD) or
 * la_backward (op = LA_OP_BACKWARD) needs for these sizes; 0 means none.
 * Returns 0 as well for arguments the calls would reject.  The amount
 * depends only on the arguments, so one buffer can be sized once and reused
 * by calls on the same stream.
 */
LA_EXPORT size_t la_workspace_size(la_op op, int64_t B, int64_t H, int64_t N, int64_t D,
                         int causal, la_dtype dt);

/*
 * Forward pass.  q, k, v (read) and o (written): [B, H, N, D] of dtype `dt`.
 * causal != 0 selects the prefix sums j <= i.  S_out [B, H, D, D] (row = key
 * feature f, column = value index) and z_out [B, H, D], float32, may each be
 * NULL; when given they receive the state after all N tokens (both modes),
 * which la_decode_step can continue from.  g_out [B, H, N], float32, may be
 * NULL; when given it receives the denominators g_i = phi(q_i) . z_i, which
 * la_backward accepts together with o to skip recomputing the forward.
 * phi_q_out, phi_k_out ([B, H, N, D] of dtype `dt`) may both be NULL; when
 * given (both) they receive phi(q) and phi(k) as the forward's products read
 * them (rounded to `dt`), which la_backward accepts to skip evaluating the
 * feature map again; one without the other is LA_ERR_INVALID_ARG.
 * Workspace: see la_workspace_size; may be NULL when that is 0.
 * Errors: LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_WORKSPACE,
 * LA_ERR_CUDA.  On error nothing has been launched except for LA_ERR_CUDA,
 * where earlier launches of the same call may have run.
 */
LA_EXPORT la_status la_forward(const void *q, const void *k, const void *v, void *o,
                     float *S_out, float *z_out, float *g_out,
                     void *phi_q_out, void *phi_k_out,
                     int64_t B, int64_t H, int64_t N, int64_t D,
                     la_dtype dt, int causal, la_phi phi,
                     void *workspace, size_t workspace_bytes, la_stream_t stream);

/*
 * Backward pass of L = sum(dO * O) for the same forward.  q, k, v, dO
 * (read) and dq, dk, dv (written): [B, H, N, D] of dtype `dt`.  o (the
 * forward's output, [B, H, N, D] of dtype `dt`) and g (the forward's g_out,
 * float32 [B, H, N]) are optional and go together: when both are NULL the
 * forward quantities are recomputed inside; when both are given they are
 * used instead (dU = dO/g and dg = -(dO . o)/g directly), which is faster.
 * phi_q, phi_k (the forward's phi_q_out, phi_k_out) are optional as well,
 * both or neither, and only together with o and g: when given, the head
 * size 64 kernels read them in place of evaluating phi on q and k (phi'
 * then comes from phi: min(phi, 1) for elu+1, 1 where phi exceeds the
 * x <= 0 value for relu+eps); other paths ignore them.
 * The tensor-core dQ products use the centred key features phi(k) - 1
 * (elu+1) so that bf16 operands keep phi's small deviations from 1; they
 * are evaluated from k, never from a saved phi(k).
 * No N x D x D tensor is ever stored: the prefix and suffix states are
 * rebuilt chunk by chunk.  dq/dk/dv must not alias the inputs.  Errors as
 * la_forward; one of o, g without the other, one of phi_q, phi_k without
 * the other, or them without o and g is LA_ERR_INVALID_ARG.
 */
LA_EXPORT la_status la_backward(const void *q, const void *k, const void *v, const void *dO,
                      const void *o, const float *g, const void *phi_q, const void *phi_k,
                      void *dq, void *dk, void *dv,
                      int64_t B, int64_t H, int64_t N, int64_t D,
                      la_dtype dt, int causal, la_phi phi,
                      void *workspace, size_t workspace_bytes, la_stream_t stream);

/*
 * One recurrent decode step for every (b, h), in place:
 *     S += phi(k) v^T,   z += phi(k),   o = S^T phi(q) / (phi(q) . z)
 * (the update comes first, so the new token attends to itself).  S: float32
 * [B, H, D, D] read and written; z: float32 [B, H, D] read and written;
 * q, k, v (read) and o (written): [B, H, D] of dtype `dt`.  A zero state is
 * a valid start (the first step then returns o = v).  o must not alias S,
 * z, q, k or v.  Errors: LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CUDA.
 */
LA_EXPORT la_status la_decode_step(float *S, float *z, const void *q, const void *k,
                         const void *v, void *o, int64_t B, int64_t H, int64_t D,
                         la_dtype dt, la_phi phi, la_stream_t stream);

/*
 * la_backward_noalloc — la_backward without a caller-provided workspace, for
 * callers that cannot allocate device memory at call time: code running
 * inside a CUDA stream capture, under a memory-pool or allocator policy that
 * forbids new allocations, or in plugins handed only their input and output
 * buffers.  The paper has no counterpart to this entry point; it exists for
 * those callers only.
 *
 * Instead of a workspace it uses one scratch array of LA_NOALLOC_MAX_BYTES
 * bytes that the library reserves statically in device memory; every GPU
 * that loads the library holds that array until the process exits.
 * Arguments and results are exactly those of la_backward.  The first call
 * on a device resolves the array's device address (a runtime call); make
 * that first call before any stream capture.  Calls whose scratch need
 * (la_workspace_size(LA_OP_BACKWARD, ...)) exceeds LA_NOALLOC_MAX_BYTES are
 * rejected with LA_ERR_WORKSPACE and nothing is launched.  All calls share
 * the one array and it keeps the last call's contents, so calls that
 * overlap on the GPU (other streams, other host threads) race: serialise
 * them.  No device memory is allocated or freed by this call.
 */
#define LA_NOALLOC_MAX_BYTES (64u << 20)

LA_EXPORT la_status la_backward_noalloc(const void *q, const void *k, const void *v,
                                        const void *dO, const void *o, const float *g,
                                        const void *phi_q, const void *phi_k,
                                        void *dq, void *dk, void *dv,
                                        int64_t B, int64_t H, int64_t N, int64_t D,
                                        la_dtype dt, int causal, la_phi phi,
                                        la_stream_t stream);

/*
 * Grouped key/value heads (grouped-query and multi-query attention, "Attention
 * Optimization", Advanced Techniques: Multi-Query Attention and Grouped-Query
 * Attention).  The same operations with Hkv key/value heads shared by the H
 * query heads: Hkv >= 1 divides H, G = H / Hkv, and query head h of batch b
 * reads k, v head h / G (heads h = 0..G-1 share head 0, and so on).  q, o,
 * dO, dq, g: [B, H, N, D] (g: [B, H, N]) as before; k, v, dk, dv:
 * [B, Hkv, N, D]; the state S_out / z_out and the decode state S, z are per
 * key/value head: [B, Hkv, D, D] and [B, Hkv, D] (the state depends on k, v
 * only); decode q and o are [B, H, D] and k, v [B, Hkv, D].  dk and dv are
 * the sums over each group's query heads (formed per query head in the
 * workspace and added in a fixed order).  The decode step updates each
 * key/value head's state once and answers the group's G queries from it, so
 * its state traffic is that of Hkv heads.  Hkv == H is exactly the call
 * without the suffix.  phi_q/phi_k (in or out) with Hkv < H is
 * LA_ERR_UNSUPPORTED; Hkv < 1 or H % Hkv != 0 is LA_ERR_INVALID_ARG.
 */
LA_EXPORT size_t la_workspace_size_gqa(la_op op, int64_t B, int64_t H, int64_t Hkv, int64_t N,
                                       int64_t D, int causal, la_dtype dt);
LA_EXPORT la_status la_forward_gqa(const void *q, const void *k, const void *v, void *o,
                                   float *S_out, float *z_out, float *g_out,
                                   void *phi_q_out, void *phi_k_out,
                                   int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t D,
                                   la_dtype dt, int causal, la_phi phi,
                                   void *workspace, size_t workspace_bytes, la_stream_t stream);
LA_EXPORT la_status la_backward_gqa(const void *q, const void *k, const void *v, const void *dO,
                                    const void *o, const float *g, const void *phi_q,
                                    const void *phi_k, void *dq, void *dk, void *dv,
                                    int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t D,
                                    la_dtype dt, int causal, la_phi phi,
                                    void *workspace, size_t workspace_bytes, la_stream_t stream);
LA_EXPORT la_status la_decode_step_gqa(float *S, float *z, const void *q, const void *k,
                                       const void *v, void *o, int64_t B, int64_t H, int64_t Hkv,
                                       int64_t D, la_dtype dt, la_phi phi, la_stream_t stream);

/*
 * Decayed (gated) linear attention, causal.  The pages name gating and decay
 * factors as the architectural change linear-attention models need to match
 * softmax quality ("Efficient Transformers Survey", Common Confusions, "Watch
 * Out: Linear attention is not a drop-in replacement") without fixing a form;
 * these calls take the plainest one, a constant factor per head:
 *     S_i = gamma_h S_{i-1} + phi(k_i) v_i^T,   z_i = gamma_h z_{i-1} + phi(k_i),
 *     o_i = S_i^T phi(q_i) / (phi(q_i) . z_i),
 * i.e. o_i averages v_j (j <= i) with weights gamma^(i-j) phi(q_i).phi(k_j).
 * gamma: HOST array of H float32 factors in [0, 1] (read during the call,
 * not kept), the same for every batch entry; gamma = 1 is the undecayed
 * causal call, gamma = 0 returns o = v.  NULL, a factor outside [0, 1] or
 * NaN is LA_ERR_INVALID_ARG; H > 256 is LA_ERR_UNSUPPORTED.  Layouts,
 * g_out, S_out / z_out (the decayed state after token N), the saved o and g
 * of la_backward_decay and the decode state are as in la_forward,
 * la_backward and la_decode_step; the decode step scales (S, z) by gamma
 * before adding the token.  There is no gradient with respect to gamma (a
 * fixed per-head constant).  la_workspace_size_decay covers every gamma.
 */
LA_EXPORT size_t la_workspace_size_decay(la_op op, int64_t B, int64_t H, int64_t N, int64_t D,
                                         la_dtype dt);
LA_EXPORT la_status la_forward_decay(const void *q, const void *k, const void *v, void *o,
                                     float *S_out, float *z_out, float *g_out,
                                     const float *gamma, int64_t B, int64_t H, int64_t N,
                                     int64_t D, la_dtype dt, la_phi phi,
                                     void *workspace, size_t workspace_bytes, la_stream_t stream);
LA_EXPORT la_status la_backward_decay(const void *q, const void *k, const void *v,
                                      const void *dO, const void *o, const float *g,
                                      void *dq, void *dk, void *dv, const float *gamma,
                                      int64_t B, int64_t H, int64_t N, int64_t D,
                                      la_dtype dt, la_phi phi,
                                      void *workspace, size_t workspace_bytes, la_stream_t stream);
LA_EXPORT la_status la_decode_step_decay(float *S, float *z, const void *q, const void *k,
                                         const void *v, void *o, const float *gamma,
                                         int64_t B, int64_t H, int64_t D, la_dtype dt, la_phi phi,
                                         la_stream_t stream);

/*
 * Performer positive random features (FAVOR+; "Efficient Transformers
 * Survey", Low-Rank Approximations, Performer, and Proposition "Performer
 * Approximation Quality"):
 *     phi(x) = m^-1/2 exp(-|x|^2 / 2) [exp(w_1^T x), ..., exp(w_m^T x)],
 * an unbiased estimate of the exponential kernel: E[phi(q)^T phi(k)] =
 * exp(q^T k).  x: [B, H, N, D] bf16 rows (q or k, pre-normalised by the
 * caller: x = q / D^(1/4) gives softmax attention's exp(q^T k / sqrt(D)));
 * omega: [m, D] bf16, row i = w_i, drawn by the caller from N(0, I_D) (the
 * random numbers are an input; one draw shared by every head); phi out:
 * [B, H, N, m] bf16.  The features feed la_forward / la_backward with phi =
 * LA_PHI_IDENTITY (q = phi(q), k = phi(k); values v of head size m).
 * la_favor_features_backward returns dx [B, H, N, D] of sum(dphi * phi(x))
 * given x, omega and dphi [B, H, N, m]: dx = sum_i dphi_i phi_i w_i -
 * x sum_i dphi_i phi_i, with phi recomputed from x in float32 (the stored
 * features are not read).  Supported: bf16 with D and m each 64 or 128 (else
 * LA_ERR_UNSUPPORTED); float32 accumulation, outputs rounded to bf16 once.
 * No workspace.  With m != D the features go to la_forward_mv /
 * la_backward_mv (feature length m, head size D).
 */
LA_EXPORT la_status la_favor_features(const void *x, const void *omega, void *phi, int64_t B,
                                      int64_t H, int64_t N, int64_t D, int64_t m, la_dtype dt,
                                      la_stream_t stream);
LA_EXPORT la_status la_favor_features_backward(const void *x, const void *omega,
                                               const void *dphi, void *dx, int64_t B, int64_t H,
                                               int64_t N, int64_t D, int64_t m, la_dtype dt,
                                               la_stream_t stream);

/*
 * Attention whose feature vectors and values differ in length: q, k
 * [B, H, N, Dk] (with LA_PHI_IDENTITY the features themselves, e.g. m = Dk
 * Performer features from la_favor_features), v, o, dO, dv [B, H, N, Dv];
 * S = sum_j phi(k_j) v_j^T is Dk x Dv ("Efficient Transformers Survey",
 * Proposition "Linear Attention via Kernel Decomposition": phi maps R^d to
 * R^m; Low-Rank Approximations, Performer).  Otherwise as la_forward /
 * la_backward (g_out, saved o and g).  bf16, Dk and Dv each 64 or 128;
 * Dk < Dv needs LA_PHI_IDENTITY (its widening zero features contribute
 * nothing; a feature map would turn them into phi(0) != 0), else
 * LA_ERR_UNSUPPORTED.  Implementation: the narrower side is widened with
 * zero columns into the workspace (values: zero output columns; features:
 * zero terms), the head-size max(Dk, Dv) kernels run, and the wider result
 * is cut back; the copies cost 2 (forward) to 4 (backward) extra passes over
 * one tensor of the wider size.  Dk == Dv is exactly la_forward /
 * la_backward.  Workspace: la_workspace_size_mv.
 */
LA_EXPORT size_t la_workspace_size_mv(la_op op, int64_t B, int64_t H, int64_t N, int64_t Dk,
                                      int64_t Dv, int causal, la_dtype dt);
LA_EXPORT la_status la_forward_mv(const void *q, const void *k, const void *v, void *o,
                                  float *g_out, int64_t B, int64_t H, int64_t N, int64_t Dk,
                                  int64_t Dv, la_dtype dt, int causal, la_phi phi,
                                  void *workspace, size_t workspace_bytes, la_stream_t stream);
LA_EXPORT la_status la_backward_mv(const void *q, const void *k, const void *v, const void *dO,
                                   const void *o, const float *g, void *dq, void *dk, void *dv,
                                   int64_t B, int64_t H, int64_t N, int64_t Dk, int64_t Dv,
                                   la_dtype dt, int causal, la_phi phi, void *workspace,
                                   size_t workspace_bytes, la_stream_t stream);

/*
 * Sequence split across ranks (one process per GPU): the N tokens of every
 * head are cut into consecutive shards, rank r holding shard r.  S and z are
 * sums over tokens ("Efficient Transformers Survey", Proposition "Linear
 * Attention via Kernel Decomposition", Statement; "Why It Matters": the
 * state is carried along the sequence), so a rank's outputs need only one
 * state record per head from the other ranks: the sum over the shards
 * before it (causal) or over all shards (non-causal); the backward needs
 * the same for the centred key features, and the sum of the query-side
 * state over the shards after it (causal) or all shards.  The calls below
 * are a rank's local steps; the caller moves the records between ranks
 * (an all-gather of one record per head per rank, e.g. NCCL) and forms the
 * incoming sums with la_state_range_sum.  Per rank and call order:
 *
 *   forward:  la_state_local(k, v, centred=0) -> rec;  all-gather rec;
 *             la_state_range_sum(lo=0, hi=rank or P) -> in;
 *             la_forward_sp(q, k, v, in) -> o, g.
 *   backward: la_state_local(k, v, centred=1) -> rec;  all-gather;
 *             la_state_range_sum(0, rank or P) -> in;
 *             la_backward_sp_dq(..., o, g, in) -> dq, rec2;  all-gather rec2;
 *             la_state_range_sum(rank+1 or 0, P) -> in2;
 *             la_backward_sp_dkdv(..., g, in2) -> dk, dv.
 *
 * A state record is float32 [D*D + D]: S [D][D] (row = key feature) then z
 * [D]; a record array is [B, H, D*D + D].  Tensors are this rank's shard,
 * [B, H, N, D] with N its token count.  Tensor-core path only: bf16 with
 * D = 64 or 128 (else LA_ERR_UNSUPPORTED), one key/value head per query
 * head, no decay.  Workspace: la_workspace_size_sp(LA_OP_FORWARD, ...) for
 * la_state_local and la_forward_sp, la_workspace_size_sp(LA_OP_BACKWARD,
 * ...) (which also serves la_state_local) for the two backward calls.
 */
LA_EXPORT size_t la_workspace_size_sp(la_op op, int64_t B, int64_t H, int64_t N, int64_t D,
                                      int causal, la_dtype dt);

/*
 * This shard's state record per head, written to state_out [B, H, D*D+D]:
 * S = sum_j (phi(k_j) - c) v_j^T, z = sum_j (phi(k_j) - c), with c = 0, or
 * with centred != 0 the constant the backward's dQ products subtract from
 * the key features (1 for elu+1, 0 otherwise; la_backward's centred
 * features).  N = 0 writes zeros.  Errors as la_forward.
 */
LA_EXPORT la_status la_state_local(const void *k, const void *v, float *state_out, int64_t B,
                                   int64_t H, int64_t N, int64_t D, la_dtype dt, la_phi phi,
                                   int centred, void *workspace, size_t workspace_bytes,
                                   la_stream_t stream);

/*
 * out[h] = sum over p in [lo, hi) of states[p][h], added in increasing p
 * (bitwise reproducible); states: [P, B, H, D*D+D] float32 (the records of
 * ranks 0..P-1 in rank order, as an all-gather leaves them), out: [B, H,
 * D*D+D].  lo == hi writes zeros (rank 0's causal prefix).  0 <= lo <= hi
 * <= P, else LA_ERR_INVALID_ARG.  out must not alias states.
 */
LA_EXPORT la_status la_state_range_sum(const float *states, int64_t P, int64_t lo, int64_t hi,
                                       float *out, int64_t B, int64_t H, int64_t D,
                                       la_stream_t stream);

/*
 * la_forward on this shard starting from state_in [B, H, D*D+D]: causal,
 * the sum of the states of the shards before (outputs then equal those of
 * the whole sequence); non-causal, the sum over every shard (the local
 * tokens' own state included).  o: [B, H, N, D]; g_out (nullable) float32
 * [B, H, N] the denominators; state_out (nullable, causal only) receives
 * state_in plus this shard's state, which is the next shard's state_in.
 */
LA_EXPORT la_status la_forward_sp(const void *q, const void *k, const void *v, void *o,
                                  const float *state_in, float *state_out, float *g_out,
                                  int64_t B, int64_t H, int64_t N, int64_t D, la_dtype dt,
                                  int causal, la_phi phi, void *workspace,
                                  size_t workspace_bytes, la_stream_t stream);

/*
 * Backward, first local step: dq of this shard, given the forward's o and g
 * (required) and state_in, the centred record sum of la_state_local(...,
 * centred=1) over the shards before (causal) or every shard (non-causal).
 * state_out [B, H, D*D+D] receives this shard's query-side record, R =
 * sum_i phi(q_i) du_i^T and r = sum_i phi(q_i) dg_i with du_i = dO_i / g_i
 * and dg_i = -(dO_i . o_i) / g_i (the suffix state of the dK, dV products).
 * The workspace keeps dg and the per-block records for la_backward_sp_dkdv:
 * pass the same workspace, unchanged, to that call.
 */
LA_EXPORT la_status la_backward_sp_dq(const void *q, const void *k, const void *v,
                                      const void *dO, const void *o, const float *g,
                                      const float *state_in, void *dq, float *state_out,
                                      int64_t B, int64_t H, int64_t N, int64_t D, la_dtype dt,
                                      int causal, la_phi phi, void *workspace,
                                      size_t workspace_bytes, la_stream_t stream);

/*
 * Backward, second local step: dk, dv of this shard, given g and state_in,
 * the sum of la_backward_sp_dq's state_out over the shards after this one
 * (causal) or every shard (non-causal), and the workspace la_backward_sp_dq
 * filled.
 */
LA_EXPORT la_status la_backward_sp_dkdv(const void *q, const void *k, const void *v,
                                        const void *dO, const float *g, const float *state_in,
                                        void *dk, void *dv, int64_t B, int64_t H, int64_t N,
                                        int64_t D, la_dtype dt, int causal, la_phi phi,
                                        void *workspace, size_t workspace_bytes,
                                        la_stream_t stream);

/* Static English text for a status code (never NULL). */
LA_EXPORT const char *la_status_string(la_status status);

/*
 * Detail of the most recent LA_ERR_CUDA returned on the calling host thread:
 * the failing step and the CUDA runtime's error name ("" if none).  The
 * string stays valid until the thread's next failing call.
 */
LA_EXPORT const char *la_last_error(void);

/*
 * Kernels that wait on other thread blocks do so for a bounded number of
 * iterations; when a wait gives up, the kernel records it in a device-side
 * error word and finishes without hanging (its outputs are then invalid).
 * This call synchronises `stream`, reads and clears that word, and returns
 * LA_ERR_DEVICE_TIMEOUT if it was set, LA_ERR_CUDA if the synchronisation
 * itself failed, LA_OK otherwise.
 */
LA_EXPORT la_status la_get_device_error(la_stream_t stream);

/*
 * Failure-detection self-test.  Launches one thread block of `nthreads`
 * threads (1..1024) that all wait, through the same bounded wait the
 * chunked kernels use, on an mbarrier that nothing arrives at.  The wait
 * gives up after its limit (1 s), records the failure in the device error
 * word (so a following la_get_device_error returns LA_ERR_DEVICE_TIMEOUT and
 * clears it), every other waiting thread leaves as soon as it sees the
 * block's abort flag, and the kernel returns: a stuck pipeline ends with an
 * error status instead of hanging the GPU.  Asynchronous on `stream`.
 * Errors: LA_ERR_INVALID_ARG (nthreads out of range), LA_ERR_CUDA.
 */
LA_EXPORT la_status la_selftest_wait_timeout(int nthreads, la_stream_t stream);

/*
 * Launch accounting.  la_launch_count() is the number of kernels this
 * library has launched since it was loaded (counted on the host at launch).
 *
 * Launch timing, for benchmarks: after la_profile_enable(1) every kernel the
 * library launches is bracketed by two CUDA events recorded on its launch
 * stream.  la_profile_collect() synchronises those events, writes up to
 * `max_entries` per-kernel aggregates (name, launches, total milliseconds)
 * to `out`, clears the records and returns the number of distinct kernels
 * (which may exceed max_entries).  la_profile_enable(0) stops recording.
 * Event bookkeeping is host-side and not thread-safe across concurrent
 * callers; it allocates no device memory.
 */
typedef struct la_profile_entry {
    char name[48];
    int64_t launches;
    double total_ms;
} la_profile_entry;

LA_EXPORT uint64_t la_launch_count(void);
LA_EXPORT void la_profile_enable(int on);
LA_EXPORT int la_profile_collect(la_profile_entry *out, int max_entries);

/* Library version (LA_API_VERSION at build time). */
LA_EXPORT int la_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LA_API_H */
