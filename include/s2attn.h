/*
 * s2attn.h — C ABI of the sm_100a S²-Attn (shifted sparse attention) library.
 *
 * The operation is LongLoRA's S²-Attn ("LongLoRA: Efficient Fine-tuning of Long-Context
 * Large Language Models", paper-graph summary page, §3.4 "S2-Attn: Shifted Sparse
 * Attention as a Training-Time Proxy for Full Attention", Algorithm 1):
 *   1. split the Hq query heads into two chunks; in the second chunk (heads
 *      [Hq/2, Hq)) roll every sequence by -G/2 along the token axis, with wrap-around
 *      (torch.roll semantics: rolled[r] = x[(r + G/2) mod N]);
 *   2. view the N tokens as N/G independent groups of G consecutive (rolled) tokens;
 *   3. inside each group apply standard causal self-attention
 *      o = softmax(scale * q k^T) v, the causal mask taken in rolled order;
 *   4. roll the second chunk's output back by +G/2.
 * The backward is the gradient of those steps (the page uses S²-Attn only during
 * fine-tuning, §3.2, so gradients flow through it).
 * Grouped-query heads: query head h reads key/value head h / (Hq / Hkv); its roll is
 * applied to that shared key/value view.
 *
 * Layouts (all row-major, contiguous, every token axis in ORIGINAL order):
 *   q, o, dO, dq : bf16 [B, N, Hq,  d]
 *   k, v, dk, dv : bf16 [B, N, Hkv, d]
 *   lse          : fp32 [B, Hq, N]   natural-log row log-sum-exp of scale * q k^T over
 *                                    the keys the row attends to
 * Pointers are device pointers (the caller's CUDA device must be current), 16-byte
 * aligned. `stream` is a cudaStream_t (NULL = legacy default stream).
 *
 * Ownership and behaviour: the caller owns every buffer. The library allocates no memory,
 * keeps no per-call state, never synchronises the stream (except
 * s2attn_get_device_error), and launches asynchronously on `stream`. Outputs are
 * overwritten, never accumulated.
 *
 * Errors: arguments are validated on the host before any launch;
 *   S2ATTN_ERR_INVALID_ARG  null / misaligned pointer, a size <= 0, Hq % Hkv != 0,
 *                           N % G != 0 (unless S2ATTN_FLAG_PARTIAL_LAST_GROUP),
 *                           odd Hq (default split), unknown option flags, scale not a
 *                           positive finite number, shift_head_begin outside [0, Hq],
 *                           workspace too small;
 *   S2ATTN_ERR_UNSUPPORTED  d not in {64, 128}; N >= 2^30;
 *   S2ATTN_ERR_CUDA         a CUDA call or a launch failed (see s2attn_last_error);
 *   S2ATTN_ERR_TIMEOUT      reported by s2attn_get_device_error: a kernel's pipeline wait
 *                           exceeded its limit; the kernel stopped early and returned
 *                           (its outputs are undefined), the context stays usable.
 */
#ifndef S2ATTN_H_
#define S2ATTN_H_

#include <stddef.h>

#if defined(__GNUC__)
#define S2ATTN_API __attribute__((visibility("default")))
#else
#define S2ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  S2ATTN_OK = 0,
  S2ATTN_ERR_INVALID_ARG = 1,
  S2ATTN_ERR_UNSUPPORTED = 2,
  S2ATTN_ERR_CUDA = 3,
  S2ATTN_ERR_TIMEOUT = 4
} s2attn_status;

/* Version of this ABI (bumped on any signature change or workspace-size change); 2 adds the
 * dS hand-off entries and the work counters in the backward workspace; 3 adds the option flags
 * (_general entries, which replace the strided-only entries) and s2attn_rope_pi; 4 adds the
 * _general forms of the two dS hand-off stages; 5 adds s2attn_fwd_rope_q. */
S2ATTN_API int s2attn_abi_version(void);

/* Static description of a status code. */
S2ATTN_API const char* s2attn_status_string(int status);

/* Text of the last CUDA error seen by the calling host thread ("" if none). */
S2ATTN_API const char* s2attn_last_error(void);

/*
 * Forward: o and lse from q, k, v (Algorithm 1: roll -> self_attn -> roll back).
 * Heads [Hq/2, Hq) are rolled by G/2 (rounded down when G is odd: the page's group of
 * 1/6 of 8192 tokens, Table 7, is G = 1365 rolled by 682). Any G >= 1 and any roll are
 * supported. scale multiplies q k^T (1/sqrt(d) for Llama2).
 */
S2ATTN_API s2attn_status s2attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int Hq, int Hkv, int N, int d, int G, float scale,
                         void* stream);

/*
 * Forward with the head split and the roll made explicit: heads
 * [shift_head_begin, Hq) are rolled so that rolled[r] = x[(r + shift) mod N].
 * s2attn_fwd == s2attn_fwd_ex(..., Hq/2, G/2, ...). shift_head_begin = Hq gives plain
 * grouped causal attention (the page's "short attention", Pattern 1 only); 0 rolls every
 * head (Pattern 2 only); shift = N - G/2 is the page's "shift up" variant (Table 8);
 * G = N with shift_head_begin = Hq is full causal attention. shift may be any integer; it
 * is taken mod N.
 */
S2ATTN_API s2attn_status s2attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int Hq, int Hkv, int N, int d, int G, float scale,
                            int shift_head_begin, int shift, void* stream);

/* Option flags of the _general entry points (at most one of the first two). */
#define S2ATTN_FLAG_WRAP_OWN_GROUP 1
#define S2ATTN_FLAG_WRAP_FRONT_FIRST 2
#define S2ATTN_FLAG_PARTIAL_LAST_GROUP 4
/*
 * S2ATTN_FLAG_WRAP_OWN_GROUP is the pages' Variant 2 (summary page, §3.4 "Information
 * leakage considerations", Table 8, Figure 6): in the rolled heads the tokens that the roll
 * wrapped around (original tokens 0..shift-1) form their own group instead of sharing the
 * last group with the last G - shift tokens, i.e. the last rolled group is split at the wrap
 * into two causal groups. Requires a rolled head (shift_head_begin < Hq) and 0 < shift < G
 * (after reduction mod N), else S2ATTN_ERR_INVALID_ARG.
 *
 * S2ATTN_FLAG_WRAP_FRONT_FIRST is the pages' Variant 3 (same passage: the shifted tokens swap
 * places with the original front tokens): in the rolled heads the last rolled group lists the
 * wrapped tokens 0..shift-1 first and the last G - shift tokens after them, so the causal
 * order inside it is the original token order (the wrapped tokens no longer see the end of the
 * sequence; the end of the sequence sees them). Same requirements as Variant 2; combining the
 * two flags is S2ATTN_ERR_INVALID_ARG.
 *
 * S2ATTN_FLAG_PARTIAL_LAST_GROUP admits N not divisible by G (summary page, Table 7, groups of
 * 1/6 of the context): the rolled sequence is cut into groups of G rows and the last group is
 * shorter (N mod G rows), which is what padding the grouped view to a multiple of G with rows
 * that no query sees amounts to. G may then exceed N (one partial group). Without the flag
 * N % G != 0 is S2ATTN_ERR_INVALID_ARG; with it and G | N it changes nothing. It cannot be
 * combined with Variant 2 or 3 when G does not divide N (S2ATTN_ERR_INVALID_ARG).
 *
 * Strides. Each [B, N, H, d] tensor X is read or written at X + b*sb + t*st + h*d + c
 * (elements): the (H, d) block of a token is contiguous, tokens and batches may be spaced
 * freely. This takes q, k and v as views of one packed qkv [B, N, 3, H, d] buffer, the layout
 * LongLoRA's Algorithm 1 (summary page, §3.4) feeds its attention: q = qkv, k = qkv + H*d,
 * v = qkv + 2*H*d, st = 3*H*d, sb = N*st (and likewise dq, dk, dv into a packed dqkv).
 * `strides` holds {sb, st} pairs: q, k, v, o for the forward; q, k, v, o, dO, dq, dk, dv for
 * the backward; NULL means contiguous. Every stride must be a multiple of 8 elements,
 * st >= H*d and, when B > 1, sb >= N*st; otherwise S2ATTN_ERR_INVALID_ARG. lse stays a
 * contiguous [B, Hq, N] array. Outputs must not overlap each other or the inputs.
 *
 * s2attn_fwd_general: s2attn_fwd_ex with option flags and strides.
 */
S2ATTN_API s2attn_status s2attn_fwd_general(const void* q, const void* k, const void* v, void* o,
                                            float* lse, int B, int Hq, int Hkv, int N, int d,
                                            int G, float scale, int shift_head_begin, int shift,
                                            int flags, const long long* strides, void* stream);

/*
 * Forward with the rotary position embedding of the queries fused into the kernel's query-tile
 * path (summary page, §3 "Phase 1" step 2 and §4 "Model setup": RoPE with positions rescaled by
 * Position Interpolation, the step just before the attention). q holds the UN-rotated queries;
 * k must already be rotated (s2attn_rope_pi); each 128-row query tile is rotated in shared
 * memory after it lands, exactly the rotation s2attn_rope_pi applies (pair (x[i], x[i + d/2]) of
 * token t turned by (t * pi_scale) * base^(-2i/d)), before the tensor cores read it, and the
 * rotated rows are also written to q_rot (contiguous bf16 [B, N, Hq, d]), which the backward
 * needs. Otherwise as s2attn_fwd_general with contiguous tensors (no strides). q_rot may be q
 * itself (rotation in place: every query row is read and rewritten by the same tile); no other
 * overlap is allowed. Errors as s2attn_fwd_general, plus: q_rot NULL or misaligned, base <= 1 or
 * pi_scale <= 0 -> S2ATTN_ERR_INVALID_ARG; N >= 2^24 -> S2ATTN_ERR_UNSUPPORTED.
 */
S2ATTN_API s2attn_status s2attn_fwd_rope_q(const void* q, const void* k, const void* v, void* o,
                                           float* lse, void* q_rot, int B, int Hq, int Hkv,
                                           int N, int d, int G, float scale,
                                           int shift_head_begin, int shift, int flags,
                                           float base, float pi_scale, void* stream);

/* Smallest device workspace s2attn_bwd accepts: two fp32 [B, Hq, N] arrays (D and LSE in
 * base 2), each rounded up to 256 bytes, and 256 bytes of work counters for the gradient
 * kernels (cleared by the preprocess). With only this much the dQ kernel recomputes S and
 * dP (three GEMMs for one gradient). */
S2ATTN_API size_t s2attn_bwd_workspace_size(int B, int Hq, int N);

/*
 * Workspace that lets s2attn_bwd skip that recomputation: the minimum above plus room for
 * the bf16 dS tiles (128 x 128, 32 KB each) that the dK/dV kernel hands to the dQ kernel,
 * one per (batch, query head, rolled query tile, original kv tile it reads) — about
 * B * Hq * (N/128) * (G/128 + 1) / 2 tiles when G and the roll are multiples of 128, and
 * B * Hq * (N/128) * (largest such count) otherwise. cap_bytes = 0 returns the size for all
 * kv heads in one pass; otherwise the largest size <= cap_bytes that holds a whole number of
 * kv heads (at least one, even if that exceeds the cap): s2attn_bwd then runs the dK/dV and
 * dQ kernels once per group of that many kv heads. Returns 0 for arguments s2attn_bwd_ex
 * would reject.
 */
S2ATTN_API size_t s2attn_bwd_workspace_size_ex(int B, int Hq, int Hkv, int N, int d, int G,
                                               int shift_head_begin, int shift, size_t cap_bytes);
/* The same for the option flags of s2attn_bwd_general (Variant 2 changes the dS tile count). */
S2ATTN_API size_t s2attn_bwd_workspace_size_general(int B, int Hq, int Hkv, int N, int d, int G,
                                                    int shift_head_begin, int shift, int flags,
                                                    size_t cap_bytes);

/*
 * Backward: dq, dk, dv from q, k, v, the forward's o and lse, and the upstream dO.
 * Runs, in order on `stream`: the preprocess D = rowsum(dO o O), then the dK/dV kernel and
 * a dQ kernel. `workspace` (device, 256-byte aligned, >= s2attn_bwd_workspace_size bytes)
 * is scratch owned by the caller; its contents on entry do not matter. If it also holds the
 * dS tiles of at least one kv head (s2attn_bwd_workspace_size_ex), the dK/dV kernel stores
 * dS there and the dQ kernel is a plain GEMM over them, repeated per group of kv heads that
 * fits; otherwise the dQ kernel recomputes S and dP. Both give the same gradients up to
 * fp32 summation order.
 * dk and dv are the sums over the query heads sharing each kv head.
 */
S2ATTN_API s2attn_status s2attn_bwd(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dO, void* dq, void* dk, void* dv,
                         int B, int Hq, int Hkv, int N, int d, int G, float scale,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Backward with explicit head split and roll (same meaning as s2attn_fwd_ex). */
S2ATTN_API s2attn_status s2attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, void* dq, void* dk, void* dv,
                            int B, int Hq, int Hkv, int N, int d, int G, float scale,
                            int shift_head_begin, int shift, void* workspace,
                            size_t workspace_bytes, void* stream);

/* s2attn_bwd_ex with option flags and strides (see s2attn_fwd_general; 8 {sb, st} pairs).
 * With flags, size the workspace with s2attn_bwd_workspace_size_general. */
S2ATTN_API s2attn_status s2attn_bwd_general(const void* q, const void* k, const void* v,
                                            const void* o, const float* lse, const void* dO,
                                            void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                                            int N, int d, int G, float scale,
                                            int shift_head_begin, int shift, int flags,
                                            const long long* strides, void* workspace,
                                            size_t workspace_bytes, void* stream);

/*
 * The three stages of s2attn_bwd, callable one at a time (same arguments; the workspace
 * must carry the preprocess results into the two gradient stages):
 *   s2attn_bwd_preprocess  workspace <- D = rowsum(dO o O) and LSE * log2(e)
 *   s2attn_bwd_dkdv        dk, dv    <- from q, k, v, dO and the workspace
 *   s2attn_bwd_dq          dq        <- from q, k, v, dO and the workspace
 * Arguments a stage does not use may be NULL.
 */
S2ATTN_API s2attn_status s2attn_bwd_preprocess(const void* o, const float* lse, const void* dO,
                                    int B, int Hq, int N, int d, void* workspace,
                                    size_t workspace_bytes, void* stream);
S2ATTN_API s2attn_status s2attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO,
                              void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int G,
                              float scale, int shift_head_begin, int shift,
                              const void* workspace, size_t workspace_bytes, void* stream);
S2ATTN_API s2attn_status s2attn_bwd_dq(const void* q, const void* k, const void* v, const void* dO,
                            void* dq, int B, int Hq, int Hkv, int N, int d, int G, float scale,
                            int shift_head_begin, int shift, const void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * The two gradient stages of the dS hand-off, one kv-head group covering all kv heads, for the
 * default variant and contiguous tensors (the _general forms below take option flags and
 * strides): the workspace must be at least s2attn_bwd_workspace_size_ex(..., cap_bytes = 0)
 * bytes, else S2ATTN_ERR_INVALID_ARG. Run s2attn_bwd_preprocess, then, on the same stream and with the
 * same workspace:
 *   s2attn_bwd_dkdv_ds  dk, dv and the dS tiles <- from q, k, v, dO and D, LSE2
 *   s2attn_bwd_dq_ds    dq                      <- from k and the dS tiles
 */
S2ATTN_API s2attn_status s2attn_bwd_dkdv_ds(const void* q, const void* k, const void* v,
                                            const void* dO, void* dk, void* dv, int B, int Hq,
                                            int Hkv, int N, int d, int G, float scale,
                                            int shift_head_begin, int shift, void* workspace,
                                            size_t workspace_bytes, void* stream);
S2ATTN_API s2attn_status s2attn_bwd_dq_ds(const void* k, void* dq, int B, int Hq, int Hkv, int N,
                                          int d, int G, float scale, int shift_head_begin,
                                          int shift, const void* workspace,
                                          size_t workspace_bytes, void* stream);

/*
 * The two dS hand-off stages with option flags and strides, so that a caller driving the
 * backward stage by stage keeps every variant of s2attn_bwd_general (Variants 2 and 3 of the
 * pages' Table 8, a shorter last group) and packed dqkv outputs. Arguments as in
 * s2attn_bwd_general: `strides` is NULL or its 8 {sb, st} pairs (q, k, v, o, dO, dq, dk, dv;
 * the pairs of tensors a stage does not touch are validated but unused). The workspace must be
 * at least s2attn_bwd_workspace_size_general(..., flags, cap_bytes = 0) bytes and carry the
 * preprocess results (s2attn_bwd_preprocess) of the same o, lse, dO; errors as in
 * s2attn_bwd_general, and S2ATTN_ERR_INVALID_ARG if the workspace holds the dS tiles of fewer
 * than all kv heads. Run s2attn_bwd_dkdv_ds_general, then s2attn_bwd_dq_ds_general, on the
 * same stream with the same flags.
 */
S2ATTN_API s2attn_status s2attn_bwd_dkdv_ds_general(const void* q, const void* k, const void* v,
                                                    const void* dO, void* dk, void* dv, int B,
                                                    int Hq, int Hkv, int N, int d, int G,
                                                    float scale, int shift_head_begin, int shift,
                                                    int flags, const long long* strides,
                                                    void* workspace, size_t workspace_bytes,
                                                    void* stream);
S2ATTN_API s2attn_status s2attn_bwd_dq_ds_general(const void* k, void* dq, int B, int Hq, int Hkv,
                                                  int N, int d, int G, float scale,
                                                  int shift_head_begin, int shift, int flags,
                                                  const long long* strides, const void* workspace,
                                                  size_t workspace_bytes, void* stream);

/*
 * Backward without a caller-provided workspace, for callers that cannot allocate device
 * memory: plugin hosts whose fixed call signature carries no scratch buffer, or code on a
 * latency-critical path that must not call cudaMalloc (which can synchronise the device and
 * can fail under memory pressure at an arbitrary point). The pages have no counterpart to
 * this entry point; it exists only for such callers.
 *
 * Same arguments and results as s2attn_bwd, minus the workspace. The scratch (D and
 * LSE * log2(e), 8 bytes per (batch, head, token) row, the work counters, and the dS tiles
 * of the dQ pass when one kv head's fit in the rest) lives in an array of 16 MiB + 256 bytes
 * compiled into the library: B * Hq * N may be at most 2,097,152, larger shapes are rejected with
 * S2ATTN_ERR_UNSUPPORTED (message in s2attn_last_error) before anything is launched. Every
 * device that loads the library holds that array until the process exits. The first call on
 * a device, with that device current, looks up the array's device address; make that first
 * call before any stream capture. Nothing is allocated, by the library or by anything it
 * calls. All calls share the one array, so two calls whose kernels overlap on the GPU (other
 * streams, other host threads) race on it and give wrong results: serialise them. Nothing in
 * the array needs to start at zero: each call overwrites what it reads.
 */
S2ATTN_API s2attn_status s2attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                            const void* o, const float* lse, const void* dO,
                                            void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                                            int N, int d, int G, float scale, void* stream);

/*
 * Synchronises `stream`, then reads and clears the current device's error word.
 * Returns S2ATTN_ERR_TIMEOUT if a kernel gave up on a pipeline wait since the last call
 * (code_out, if not NULL, receives (kernel << 8) | wait site; 0 if none), S2ATTN_ERR_CUDA
 * if the synchronisation failed, S2ATTN_OK otherwise.
 */
S2ATTN_API s2attn_status s2attn_get_device_error(void* stream, unsigned int* code_out);

/* Limit on every pipeline wait inside the kernels, in nanoseconds (default 1e9). Applies
 * to launches made after the call, from any thread. 0 restores the default. */
S2ATTN_API void s2attn_set_wait_timeout_ns(unsigned long long ns);

/*
 * Failure-detection self test: launches one CTA that waits, with the same bounded wait the
 * attention kernels use, on a barrier nothing ever arrives on. After `timeout_ns` the wait
 * gives up and records an error, so the following s2attn_get_device_error returns
 * S2ATTN_ERR_TIMEOUT. No fault, trap or hang is involved.
 */
S2ATTN_API s2attn_status s2attn_selftest_wait_timeout(unsigned long long timeout_ns, void* stream);

/*
 * Rotary position embedding with Position Interpolation: the step just before the attention
 * (summary page, §3 "Phase 1" step 2, and §4 "Model setup": RoPE with positions rescaled by
 * Position Interpolation). x and y are bf16 [B, N, H, d] (d = 64 or 128); for token t and
 * i < d/2 the pair (x[.., i], x[.., i + d/2]) is turned by the angle (t * pi_scale) *
 * base^(-2i/d) (the Llama half-split pairing; t in original order) and written to y.
 * pi_scale is the Position Interpolation factor (pre-trained context / extended context, e.g.
 * 4096/8192 = 0.5; 1 for plain RoPE); base is the frequency base (10000 for Llama 2).
 * inverse = 1 turns by the opposite angle: the transpose of the rotation, which maps dq, dk
 * with respect to the rotated q, k back to the unrotated ones.
 * y == x (in place) is allowed; other overlaps are not. `strides` = NULL (contiguous) or
 * {x_sb, x_st, y_sb, y_st} in elements, with the rules of s2attn_fwd_general (so q and k can
 * be rotated inside a packed qkv buffer). Errors: null or misaligned pointers, B, N, H <= 0,
 * base <= 1, pi_scale <= 0, inverse not 0/1, bad strides -> S2ATTN_ERR_INVALID_ARG;
 * d not in {64, 128}, N >= 2^24 -> S2ATTN_ERR_UNSUPPORTED; launch failure -> S2ATTN_ERR_CUDA.
 * Asynchronous on `stream`; allocates nothing.
 */
S2ATTN_API s2attn_status s2attn_rope_pi(const void* x, void* y, int B, int N, int H, int d,
                                        float base, float pi_scale, int inverse,
                                        const long long* strides, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* S2ATTN_H_ */
