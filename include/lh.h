/*
 * lh.h - C ABI of the Lighthouse selection layer on NVIDIA B200 (sm_100a).
 *
 * The layer wraps causal scaled-dot-product attention in five steps. It builds a symmetric
 * average-pooling pyramid over Q, K and V. It scores every cell with the l2 norms of its query
 * and key, max-pooled up the levels. It picks a stratified top-K that always keeps the coarsest
 * level. It gathers the picks into one short causal subsequence and runs dense causal attention
 * on it. Finally it scatters the outputs back to token positions. The backward pass sends
 * gradients to Q, K and V through the scatter, the attention and the gather; the selection gets
 * none.
 *
 * Sources: "Long Context Pre-Training with Lighthouse Attention" (gist.science summary),
 * technical summary sections 2.A (pyramid), 2.B (scoring, selection, no gradient through the
 * selection), 2.C (gather, dense attention, scatter-back), 2.D (recovery phase = dense SDPA);
 * and the Nous Research article on edge.aivizor.me, the paragraph listing the four stages
 * ("two scalar scores per cell", "the coarsest level is always kept").
 *
 * Conventions common to every entry point:
 *  - Tensors are contiguous [B, H, rows, d] with d fastest. They live in device memory that the
 *    caller allocates and frees. The library never allocates, frees or synchronises, except for
 *    lh_check, which synchronises the stream it is given.
 *  - The element type of Q, K, V, pyramid, q/k/v/do_sub and output tensors is shape.dtype (fp32
 *    or bf16). Score, lse, o_sub and the sub-gradients dq_sub/dk_sub/dv_sub are always fp32.
 *  - `stream` is a cudaStream_t passed as void*. NULL means the legacy default stream. Every
 *    launch is asynchronous and stream-ordered.
 *  - Return values report host-side validation and launch errors. Nothing is launched when
 *    validation fails. Device-side faults that the kernels detect (an out-of-range row id, a
 *    bounded wait that ran out) set a status word in the workspace; lh_check reports it.
 *  - Every device pointer must be 16-byte aligned; otherwise LH_ERR_INVALID_ARG.
 *  - Row ids (idx) are int32 ids into the concatenated pyramid of each (b, h): tokens have ids
 *    0..N-1; cell j of level l >= 1 has id N + off_l + j with off_l = sum_{l'=1}^{l-1} N/p^l'.
 *    Levels 1..L-1 are stored in one [B, H, R, d] tensor per X in Q, K, V, level 1 first.
 *  - Numerics: fp32 accumulation everywhere; scores in one fixed fp32 order (16-byte groups of
 *    separately rounded squares in ascending order, a halving tree over the groups, a correctly
 *    rounded square root) so that the selection is reproducible bit for bit; one rounding to the
 *    storage dtype.
 */
#ifndef LIGHTHOUSE_LH_H
#define LIGHTHOUSE_LH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LH_OK = 0,
  LH_ERR_INVALID_ARG = 1,  /* bad shape, null or misaligned pointer */
  LH_ERR_UNSUPPORTED = 2,  /* valid for the method but not for this GPU path (e.g. d not 64/128) */
  LH_ERR_WORKSPACE = 3,    /* workspace too small */
  LH_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
  LH_ERR_DEVICE = 5        /* a kernel reported a fault through the workspace status word */
} lh_status;

typedef enum { LH_F32 = 0, LH_BF16 = 1 } lh_dtype;

/* lh_shape.flags */
#define LH_DETERMINISTIC 1 /* attention backward without atomics: bit-identical results run to run */

/* One layer call. Names follow the pages: N tokens, H heads, d = d_head, pooling factor p,
 * L levels, S = subsequence length (the top-K budget plus the kept coarsest cells).
 * The softmax scale is fixed to 1/sqrt(d).
 * flags: 0 or LH_DETERMINISTIC. The default attention backward computes dK, dV and dQ in one
 * pass over the key blocks and adds the per-block dQ terms into dq_sub with fp32 reductions
 * (atomic adds at d = 128, copy-engine tensor reductions at d = 64), whose order varies from
 * run to run (so do the last bits of dQ). With LH_DETERMINISTIC it runs a second pass for dQ
 * instead (no atomics; slower). Everything else is deterministic either way.
 * Hkv: key/value heads (grouped-query attention; the pages state no such model, this is a
 * reading). 0 means Hkv = H. Otherwise H must be a multiple of Hkv: query head h then uses
 * key/value head h / (H / Hkv). K, V, their pyramid levels and dK, dV have Hkv heads; Q, O,
 * the scores, the selection, the subsequence (q_sub, k_sub, v_sub) and dQ have H: every
 * query head selects its own cells, and its k_sub / v_sub rows come from its key/value head.
 * A key/value head's dK and dV add the terms of its H / Hkv query heads (coarsest level
 * first, ascending heads within a level). */
typedef struct {
  int B, H, N, d, p, L, S;
  int dtype; /* lh_dtype */
  int flags;
  int Hkv;
} lh_shape;

/* Sizes derived from a shape (the pages' notation: p, L, N per level, budget S).
 * The selection is stratified: a stratum is a run of G consecutive chunks, the fewest over
 * which the budget S divides evenly (G = C / gcd(S, C); G = 1, one chunk, whenever S is a
 * multiple of C). Each stratum keeps its G coarsest cells and picks k more among its G*M
 * candidates. */
typedef struct {
  int64_t R;  /* pooled rows per (b,h): sum_{l=1}^{L-1} N/p^l */
  int64_t C;  /* chunks = coarsest cells = N/p^(L-1) */
  int64_t T;  /* tokens per chunk = p^(L-1) */
  int64_t m;  /* subsequence rows per stratum = S*G/C */
  int64_t k;  /* selected entries per stratum besides its G coarsest cells = m-G */
  int64_t M;  /* candidates per chunk = sum_{l=0}^{L-2} p^(L-1-l) */
  int64_t G;  /* chunks per stratum = C/gcd(S, C) */
} lh_sizes;

const char* lh_status_string(int status);
const char* lh_version(void);

/* Validates a shape for the GPU path and fills `out` (may be NULL).
 * Method constraints (LH_ERR_INVALID_ARG): B, H, N, d, S >= 1, p >= 2, L >= 1, dtype f32 or
 *   bf16, flags 0 or LH_DETERMINISTIC, N % p^(L-1) == 0, C <= S <= C*(M+1) (every coarsest
 *   cell kept, at most every cell).
 * GPU constraints (LH_ERR_UNSUPPORTED): d in {64, 128}; p <= 16; L <= 12; p^(L-1) <= 2^20;
 *   B*H <= 65535; N + R < 2^31; (G*M + k) * 8 + G * 4 <= 200 KiB, because a stratum's
 *   candidate keys are ranked in shared memory (at p = 4 and G = 1 this allows L <= 8);
 *   G * p^(L-1) < 2^24. */
int lh_validate(const lh_shape* shape, lh_sizes* out);

/* Bytes of the workspace `ws` that the entry points below take. The first 256 bytes hold the
 * device status word; clear them once (lh_workspace_init) before first use. */
size_t lh_workspace_bytes(const lh_shape* shape);
/* Bytes of the forward-to-backward context `saved` of lh_layer_fwd / lh_layer_bwd. */
size_t lh_saved_bytes(const lh_shape* shape);

/* Clears the status word of `ws` (stream-ordered). */
int lh_workspace_init(void* ws, void* stream);
/* Synchronises `stream`, reads and clears the status word of `ws`.
 * Returns LH_OK or LH_ERR_DEVICE (then *flags, if non-NULL, holds the fault bits:
 * 1 = row id out of range, 2 = bounded wait ran out, 4 = after that, a wait for the kernel's own
 * copies or MMAs in flight ran out too). After flag 2 the affected outputs are unspecified;
 * the device context stays usable. */
int lh_check(void* ws, void* stream, uint32_t* flags);

/* Sets the bound of every wait inside the tensor-core kernels (a pipeline stage that never
 * arrives, for instance): after `ns` nanoseconds the kernel sets status flag 2, drains its own
 * operations in flight and returns. 0 restores the default of 2 s. Applies to launches made
 * after the call, from any thread. Returns the previous bound. Not part of the method: a
 * failure-detection control. */
uint64_t lh_set_wait_limit_ns(uint64_t ns);

/* Step 1+2 (pyramid, section 2.A; scores, section 2.B). Reads q, k, v [B,H,N,d]; writes the
 * pooled levels pq, pk, pv [B,H,R,d]. If `score` is non-NULL it also writes the rank score
 * r = max-pooled |q| + max-pooled |k| for every row id, float [B,H,N+R], in the same pass.
 * With grouped heads (shape.Hkv < H) k, v, pk, pv have Hkv heads; a first pass pools them and
 * leaves the key norms in the workspace, a second pools q and adds them to the scores.
 * pq/pk/pv may all be NULL to compute only the score (then v is not read). */
int lh_build_pyramid(const lh_shape* shape, const void* q, const void* k, const void* v,
                     void* pq, void* pk, void* pv, float* score, void* ws, void* stream);

/* Step 2 alone: the rank score float [B,H,N+R] from q [B,H,N,d] and k [B,Hkv,N,d]. */
int lh_score(const lh_shape* shape, const void* q, const void* k, float* score, void* ws,
             void* stream);

/* Step 3 (stratified top-K, section 2.B and the article's four-stage paragraph). Per (b,h) and
 * stratum (G chunks, see lh_sizes): keep the G coarsest cells and the k best candidates by
 * (r desc, level desc, position asc); write their row ids in causal order (end asc, then level
 * asc) to idx int32 [B,H,S], stratum after stratum (m rows each). The rows of one chunk are then
 * contiguous and end with its coarsest cell. */
int lh_select_topk(const lh_shape* shape, const float* score, int32_t* idx, void* stream);

/* Step 4 (gather, section 2.C). x_sub[b,h,i] = row idx[b,h,i] of [x | px]. Any idx whose ids
 * are in range is accepted; out-of-range ids give zero rows and set status bit 1. With grouped
 * heads k_sub and v_sub rows of query head h come from key/value head h / (H / Hkv). */
int lh_gather(const lh_shape* shape, const void* q, const void* k, const void* v,
              const void* pq, const void* pk, const void* pv, const int32_t* idx,
              void* q_sub, void* k_sub, void* v_sub, void* ws, void* stream);

/* Step 5 (dense causal attention on the subsequence, section 2.C). Row j is visible to row i
 * iff j <= i. Writes o_sub float [B,H,S,d] (kept in fp32: the scatter-back and the backward's
 * D_i = do_sub[i] . o_sub[i] use the unrounded output) and lse float [B,H,S] (natural log). */
int lh_attn_fwd(const lh_shape* shape, const void* q_sub, const void* k_sub, const void* v_sub,
                float* o_sub, float* lse, void* ws, void* stream);

/* Backward of step 5. o_sub is float (from lh_attn_fwd); do_sub is [B,H,S,d] in shape.dtype;
 * dq_sub, dk_sub, dv_sub are float [B,H,S,d]. Uses the workspace for D_i = do_sub[i].o_sub[i]. */
int lh_attn_bwd(const lh_shape* shape, const void* q_sub, const void* k_sub, const void* v_sub,
                const float* o_sub, const float* lse, const void* do_sub, float* dq_sub,
                float* dk_sub, float* dv_sub, void* ws, void* stream);

/* Context parallelism: one rank's share of steps 5 and its backward, when a sequence is split
 * over ranks by tokens ("Long Context Pre-Training with Lighthouse Attention", technical summary
 * section 4: 1M tokens on 32 GPUs with context parallelism). `shape` is the rank's problem (its
 * tokens and its shape->S subsequence rows). Its query rows are the global rows
 * row0 .. row0 + S - 1 of the whole subsequence; k_seen and v_seen hold the global rows
 * 0 .. row0 + S - 1 (row0 + S rows per (b,h), gathered from the ranks). The causal rule is on
 * global rows.
 *  - lh_attn_fwd_cp writes o_sub and lse for the rank's rows ([B,H,S,d], [B,H,S]).
 *  - lh_attn_bwd_cp writes dq_sub for the rank's rows and dk_seen, dv_seen with row0 + S rows
 *    per (b,h): the rank's part of dK_sub and dV_sub, which the caller sums over the ranks.
 *    Like lh_attn_bwd without LH_DETERMINISTIC, dq_sub's fp32 sums arrive in varying order.
 *  - bf16 and d = 128 only, row0 and S multiples of 128: otherwise LH_ERR_UNSUPPORTED.
 *    row0 = 0 computes what lh_attn_fwd / lh_attn_bwd compute.
 * Other arguments, layouts and errors as lh_attn_fwd / lh_attn_bwd. */
int lh_attn_fwd_cp(const lh_shape* shape, int64_t row0, const void* q_sub, const void* k_seen,
                   const void* v_seen, float* o_sub, float* lse, void* ws, void* stream);
int lh_attn_bwd_cp(const lh_shape* shape, int64_t row0, const void* q_sub, const void* k_seen,
                   const void* v_seen, const float* o_sub, const float* lse, const void* do_sub,
                   float* dq_sub, float* dk_seen, float* dv_seen, void* ws, void* stream);

/* Step 6 (deterministic scatter-back, section 2.C). o[t] = sum of o_sub[i] over the rows i of
 * t's stratum whose span covers t, coarsest first, no atomics. idx must be a valid selection
 * (rows of stratum s at s*m .. s*m+m-1, each cell at most once). o_sub is float [B,H,S,d]. */
int lh_scatter(const lh_shape* shape, const int32_t* idx, const float* o_sub, void* o,
               void* stream);

/* Backward of step 6: do_sub[i] = sum of d_o over the tokens of span(i). */
int lh_scatter_bwd(const lh_shape* shape, const int32_t* idx, const void* d_o, void* do_sub,
                   void* ws, void* stream);

/* Backward of steps 1+4: dx[t] = sum over rows i covering t of dx_sub[i] / p^level(i), for
 * x in q, k, v. dx_sub are float [B,H,S,d]; dq, dk, dv are [B,H,N,d] in shape.dtype. With
 * grouped heads dk, dv are [B,Hkv,N,d]: each adds the terms of its query heads in one fp32
 * sum, from the coarsest level down and within a level in ascending head order (two launches). */
int lh_gather_bwd(const lh_shape* shape, const int32_t* idx, const float* dq_sub,
                  const float* dk_sub, const float* dv_sub, void* dq, void* dk, void* dv,
                  void* stream);

/* The whole layer forward: steps 1-6. Writes o [B,H,N,d] and the context `saved`
 * (lh_saved_bytes) that lh_layer_bwd reads: idx, q_sub, k_sub, v_sub, o_sub, lse. */
int lh_layer_fwd(const lh_shape* shape, const void* q, const void* k, const void* v, void* o,
                 void* saved, void* ws, void* stream);

/* The whole layer backward. Reads `saved` from lh_layer_fwd and d_o [B,H,N,d]; writes
 * dq, dk, dv [B,H,N,d] (dk, dv [B,Hkv,N,d] with grouped heads). */
int lh_layer_bwd(const lh_shape* shape, const void* saved, const void* d_o, void* dq, void* dk,
                 void* dv, void* ws, void* stream);

/* lh_attn_bwd without a workspace argument, for callers that cannot allocate device memory:
 * a plugin whose host framework owns every device allocation, or code that must not call the
 * allocator at all. The paper has no counterpart; this is a deployment variant of the same
 * kernels, with the same results as lh_attn_bwd.
 *  - The per-row scratch (D_i = do_sub[i] . o_sub[i]) lives in a file-scope device array of
 *    256 + 4 * LH_STATIC_SCRATCH_ROWS bytes (about 4 MiB). Every GPU that loads the library
 *    holds it until the process exits. The call itself allocates and frees nothing.
 *  - The first call on a device (or of lh_check_static) looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current and clears its status word with a
 *    synchronous memset. Make that first call before any stream capture.
 *  - Returns LH_ERR_WORKSPACE, launching nothing, when B*H*S > LH_STATIC_SCRATCH_ROWS.
 *  - All calls share the one array, which keeps the previous call's contents. D is rewritten
 *    in full by every call before it is read. Calls that overlap on the GPU (different
 *    streams, no ordering between them) race on it.
 *  - Device faults (bounded wait ran out) latch in the array's status word; lh_check_static
 *    reads and clears it.
 *  - Other arguments, layouts and errors as lh_attn_bwd. */
#define LH_STATIC_SCRATCH_ROWS (1 << 20)
int lh_attn_bwd_static(const lh_shape* shape, const void* q_sub, const void* k_sub,
                       const void* v_sub, const float* o_sub, const float* lse,
                       const void* do_sub, float* dq_sub, float* dk_sub, float* dv_sub,
                       void* stream);
/* The status word of lh_attn_bwd_static's static scratch on the current device: synchronises
 * `stream`, reads and clears the word. Returns LH_OK or LH_ERR_DEVICE (then *flags, if
 * non-NULL, holds the fault bits as in lh_check). Allocates nothing. */
int lh_check_static(void* stream, uint32_t* flags);

/* Number of kernel launches one lh_layer_fwd (*fwd) and one lh_layer_bwd (*bwd) make for this
 * shape (either pointer may be NULL). Host-side plan only; launches nothing. */
int lh_launches(const lh_shape* shape, int* fwd, int* bwd);

/* Offsets (bytes) of the tensors inside `saved`, so that callers can read them:
 * idx, q_sub, k_sub, v_sub, o_sub, lse, in that order. */
int lh_saved_offsets(const lh_shape* shape, size_t offsets[6]);

#ifdef __cplusplus
}
#endif
#endif /* LIGHTHOUSE_LH_H */
