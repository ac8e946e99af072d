/*
 * spec_verify.h -- C ABI of libspecverify.so, the B200 (sm_100a) library for
 * the verify-and-accept step of speculative decoding.
 *
 * The step turns the target model's logits over a block of k drafted tokens
 * (plus one more position) into an accepted length and the tokens to commit.
 * "Accelerating Sonar through speculation" (Perplexity), section
 * "Speculative decoding", stages "Acceptance" and "Target generation": the
 * target runs over the draft, the longest acceptable prefix is found, and
 * the target logits at the first mismatch, or after the last draft, give one
 * more token, so n drafted tokens commit up to n + 1.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument except those named "host" is a DEVICE pointer
 *    owned by the caller.  The library allocates nothing and frees nothing.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *    default stream.  Calls only enqueue work on it and never synchronise,
 *    except spec_verify_read_device_status, which says so.
 *  - Logit tensors are row-major with the vocabulary axis contiguous; the
 *    other axes take strides in ELEMENTS (>= 0; 0 broadcasts one row).
 *    Row starts that are all 16-byte aligned take the bulk-copy (TMA) path;
 *    any other alignment takes a plain-load path with the same results.
 *  - Token and output tensors are contiguous int32.
 *  - Limits: 0 <= k <= 32, 1 <= V < 2^31, 1 <= G <= 64, B >= 0 (B = 0 is a
 *    no-op).  Every row must hold at least one finite logit; -inf is allowed,
 *    +inf and NaN are not valid logits.
 *  - The return value reports host-side validation and launch errors only
 *    (sv_status).  Errors seen on the device are recorded in the workspace
 *    and read with spec_verify_read_device_status.
 *  - Workspace: a caller-owned device buffer of at least
 *    spec_verify_workspace_size(B, G, k, V) bytes, 16-byte aligned, zeroed
 *    once (spec_verify_workspace_init) before its first use.  Each call
 *    leaves it zeroed again except for the sticky device status word.  One
 *    workspace must not be used by two calls that may run at the same time.
 *    After SV_FLAG_TIMEOUT has been reported, re-initialise it.
 */
#ifndef SPEC_VERIFY_H
#define SPEC_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Logit element types. */
typedef enum { SV_F32 = 0, SV_BF16 = 1 } sv_dtype;

/* Host-side return codes. */
typedef enum {
    SV_OK = 0,
    SV_ERR_INVALID_ARG = 1,    /* null pointer, size out of range, bad dtype or temperature */
    SV_ERR_MISALIGNED = 2,     /* pointer not aligned to its element size / workspace not 16-B */
    SV_ERR_WORKSPACE = 3,      /* workspace_bytes smaller than spec_verify_workspace_size */
    SV_ERR_CUDA = 4,           /* a CUDA runtime call or kernel launch failed */
    SV_ERR_DEVICE_TIMEOUT = 5  /* reported through the device status word only */
} sv_status;

/* Bits of the sticky device status word. */
#define SV_FLAG_INVALID_TOKEN 1u     /* a draft token was outside [0, V); it was rejected */
#define SV_FLAG_RESIDUAL_FALLBACK 2u /* no positive residual mass; correction drawn from p_n */
#define SV_FLAG_TIMEOUT 4u           /* a bounded device wait gave up; outputs are invalid */
#define SV_FLAG_INVALID_ROW 8u       /* a row map entry was outside [0, R); see the rows form */
#define SV_FLAG_CAPACITY 16u         /* spec_verify_commit: a token buffer was full */
#define SV_FLAG_INVALID_TREE 32u     /* a tree node's parent was outside [0, node) */
#define SV_FLAG_BOUNDS 64u           /* bounds-checked builds (SV_DEBUG_BOUNDS) only: a
                                        kernel formed an index outside its buffer; the
                                        access was skipped and the outputs are invalid */

/*
 * Bytes of workspace that calls with these sizes need (any mode, any dtype).
 * Returns 0 for sizes outside the limits above.
 */
size_t spec_verify_workspace_size(int B, int G, int k, int V);

/* Static, human-readable name of an sv_status value. */
const char *spec_verify_status_string(int status);

/*
 * Number of kernels this library has launched in this process, on any device
 * and stream, counted when the launch call returned success.  A launch made
 * while a stream is captured into a CUDA graph counts once, at capture, not
 * at each replay.  Calls launch: stochastic 1; greedy, multi-candidate and
 * multi-candidate rows 1 or 2 (calls of up to 512 MB of target logits stream
 * the rows in one grid and finalize in a second); threshold and tree greedy
 * 1; tree stochastic 3; commit 1; Philox 1.  Thread-safe; never fails.
 */
unsigned long long spec_verify_kernel_launches(void);

/*
 * Zero a workspace (cudaMemsetAsync on `stream`).  Needed once after the
 * buffer is allocated and again after a device timeout.
 */
int spec_verify_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Copy the sticky device status word (SV_FLAG_* bits) into *flags_host and,
 * if `clear` is nonzero, reset it.  SYNCHRONISES `stream`.
 */
int spec_verify_read_device_status(void *workspace, uint32_t *flags_host, int clear,
                                   void *stream);

/*
 * Stochastic verify (speculative rejection sampling).
 *
 * "Accelerating Sonar through speculation", section "Draft-Target":
 * acceptance compares the full draft and target probability distributions,
 * and the one logits set that the target emits after the accepted prefix is
 * sampled for the next token.  The pages give no formula; the library
 * implements the rejection-sampling rule of speculative sampling
 * (Leviathan et al. 2023; Chen et al. 2023), which keeps the output law equal
 * to the target's:
 *   p_i = softmax(target[b,i,:] / T), q_i = softmax(draft[b,i,:] / T)
 *   accept draft token x_i while u_i * q_i(x_i) < p_i(x_i)  (u_i < min(1, p/q))
 *   n = first rejected position (or k)
 *   n < k: token ~ normalize(max(0, p_n - q_n)); n = k: token ~ p_k
 * Both draws are Gumbel-max over Philox4x32-10 noise (Salmon et al., SC'11)
 * keyed by key = (seed lo, seed hi) and counter = (x >> 2, position,
 * b + seq_offset, tag), word x & 3; tags ACCEPT = 0 (c0 = 0, word 0),
 * CORRECTION = 1, BONUS = 2.  u_i = (w >> 8) 2^-24; Gumbel noise
 * g = -ln(-ln(((w >> 9) + 0.5) 2^-23)).
 *
 * target_logits  [B, k+1, V], element (b,i,x) at b*t_stride_b + i*t_stride_pos + x
 * draft_logits   [B, k, V],   element (b,i,x) at b*d_stride_b + i*d_stride_pos + x
 * draft_tokens   [B, k] int32 (a token outside [0,V) is rejected and flagged)
 * temperature    T > 0 and finite, applied to both target and draft
 * seq_offset     added to b in the Philox counter (lets a sharded batch
 *                reproduce the unsharded draws)
 * accepted_len   [B] out: n in [0, k]
 * out_tokens     [B, k+1] out: drafts 0..n-1, the sampled token at n, -1 after
 * probs_out      [B, k, 2] out, may be NULL: p_i(x_i), q_i(x_i) (0 for an
 *                invalid token) for every position up to the first
 *                rejection; a later position holds either its values or
 *                (-1, -1), when its rows were retired without being read
 *
 * Rows past a known rejection decide nothing, so the kernel does not read
 * them: positions are scheduled position by position over the batch, and a
 * chunk of row pair i of a sequence that already has a rejection before i is
 * retired unread.  The results are the same bits either way.
 */
int spec_verify_stochastic(const void *target_logits, int t_dtype, int64_t t_stride_b,
                           int64_t t_stride_pos, const void *draft_logits, int d_dtype,
                           int64_t d_stride_b, int64_t d_stride_pos,
                           const int32_t *draft_tokens, int B, int k, int V,
                           float temperature, uint64_t seed, uint32_t seq_offset,
                           int32_t *accepted_len, int32_t *out_tokens, float *probs_out,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * Greedy verify.
 *
 * "Accelerating Sonar through speculation", section "Speculative decoding":
 * the longest acceptable prefix of the draft is kept and the target gives the
 * next token for free.  Greedy acceptance: draft token i is accepted while it
 * equals argmax_x target[b,i,x] (first maximum; -0 == +0).
 *
 * target_logits [B, k+1, V] (strides as above), draft_tokens [B, k];
 * accepted_len [B] out; out_tokens [B, k+1] out: drafts 0..n-1, the argmax
 * of row n at n, -1 after.  A draft token outside [0, V) never matches and
 * raises SV_FLAG_INVALID_TOKEN (as it does in spec_verify_multi_candidate).
 */
int spec_verify_greedy(const void *target_logits, int t_dtype, int64_t t_stride_b,
                       int64_t t_stride_pos, const int32_t *draft_tokens, int B, int k, int V,
                       int32_t *accepted_len, int32_t *out_tokens, void *workspace,
                       size_t workspace_bytes, void *stream);

/*
 * Threshold acceptance (a lossy variant).
 *
 * "Accelerating Sonar through speculation", section "Speculative decoding":
 * every candidate prefix is scored by probability and the longest one at or
 * above an acceptance threshold is selected; the target gives the next token.
 * The score of the prefix of length j is its probability under the target,
 * prod_{i<j} p_i(x_i) with p_i = softmax(target[b,i,:] / temperature); the
 * accepted length n is the largest j <= k whose score is >= threshold (the
 * empty prefix scores 1), and out_tokens[b, n] is the argmax of target row n
 * (first maximum).  A draft token outside [0, V) has probability 0.  The
 * pages fix no threshold: the caller passes it, 0 < threshold <= 1.
 *
 * Arguments, layouts, outputs and workspace as spec_verify_greedy, plus
 * temperature (> 0, finite, as for spec_verify_stochastic) and threshold;
 * anything else is SV_ERR_INVALID_ARG.
 */
int spec_verify_threshold(const void *target_logits, int t_dtype, int64_t t_stride_b,
                          int64_t t_stride_pos, const int32_t *draft_tokens, int B, int k, int V,
                          float temperature, float threshold, int32_t *accepted_len,
                          int32_t *out_tokens, void *workspace, size_t workspace_bytes,
                          void *stream);

/*
 * Multi-candidate (lookahead / Jacobi n-gram) greedy verify.
 *
 * "Lookahead decoding" news piece, section "Lookahead decoding breaks the
 * order dependency" and steps 3-4: captured n-grams are validated against
 * the target and the longest accepted one is appended.  Branch g of sequence
 * b has its own rows target[b,g,0..k,:]; its accepted length n_g is its
 * longest prefix equal to the row argmaxes; the chosen branch is the longest
 * (lowest g on a tie; branch 0 when all are empty).
 *
 * target_logits [B, G, k+1, V], element (b,g,i,x) at
 *   b*t_stride_b + g*t_stride_g + i*t_stride_pos + x
 * cand_tokens [B, G, k]; best_candidate [B], accepted_len [B],
 * out_tokens [B, k+1] out (candidate g*'s first n tokens, then the argmax of
 * its row n, then -1).
 */
int spec_verify_multi_candidate(const void *target_logits, int t_dtype, int64_t t_stride_b,
                                int64_t t_stride_g, int64_t t_stride_pos,
                                const int32_t *cand_tokens, int B, int G, int k, int V,
                                int32_t *best_candidate, int32_t *accepted_len,
                                int32_t *out_tokens, void *workspace, size_t workspace_bytes,
                                void *stream);

/*
 * Multi-candidate greedy verify on deduplicated rows.
 *
 * "Lookahead decoding" news piece, steps 3-4: one decoding step verifies many
 * captured n-grams at once (the verification branch of the 2-in-1 attention
 * mask).  Candidates that share a prefix share the target rows of that prefix
 * (row i of a branch conditions on the context plus its first i tokens), so a
 * caller that evaluates each distinct prefix once passes the distinct rows and
 * a map instead of G(k+1) rows per sequence; each distinct row is then read
 * once.
 *
 * Results are exactly those of spec_verify_multi_candidate on the expanded
 * logits E[b,g,i,:] = row_logits[b, row_of[b,g,i], :].
 *
 * row_logits [B, R, V], element (b,r,x) at b*r_stride_b + r*r_stride_row + x;
 * row_of [B, G, k+1] int32 in [0, R); cand_tokens [B, G, k]; outputs as in
 * spec_verify_multi_candidate.  Requires 1 <= R <= G*(k+1) (so the workspace
 * of spec_verify_workspace_size(B, G, k, V) suffices), else
 * SV_ERR_INVALID_ARG.  A map entry outside [0, R) is not read through: that
 * row counts as one whose argmax is -1 (no candidate token matches it, and a
 * branch that stops there commits -1), and the device flag
 * SV_FLAG_INVALID_ROW is set.
 */
int spec_verify_multi_candidate_rows(const void *row_logits, int t_dtype, int64_t r_stride_b,
                                     int64_t r_stride_row, const int32_t *row_of,
                                     const int32_t *cand_tokens, int B, int G, int k, int R,
                                     int V, int32_t *best_candidate, int32_t *accepted_len,
                                     int32_t *out_tokens, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * Greedy verify of a draft token tree (EAGLE-style tree drafting).
 *
 * "Accelerating Sonar through speculation", section "EAGLE": the draft
 * explores a tree of likely tokens (Top-K candidates per node, fixed or
 * dynamically shaped), the drafted sequences are scored, the longest
 * acceptable one is kept, and one more token comes from the target.  Greedy
 * acceptance: starting at the root, the walk moves to the child whose token
 * equals the argmax of the current node's target row (first maximum; the
 * lowest-index such child if several share the token), until no child
 * matches; the target's argmax at the last node is the extra token.
 *
 * node_logits [B, N, V], element (b,j,x) at b*stride_b + j*stride_node + x:
 *   row j is the target's distribution after the path to node j (node 0 is
 *   the root: the last committed token).
 * parent [B, N] int32: parent[b][0] is ignored; parent[b][j] in [0, j) for
 *   j >= 1 (nodes in topological order).  A node whose parent is outside
 *   [0, j) is never entered, and SV_FLAG_INVALID_TREE is set.
 * tokens [B, N] int32: the draft token of node j (node 0's is ignored).
 * Outputs: accepted_len [B] = n, the accepted nodes below the root;
 *   path [B, N] = 0, then the n accepted nodes in order, then -1;
 *   out_tokens [B, N] = their n tokens, then the argmax of the last accepted
 *   node's row, then -1.
 * 1 <= N <= 64.  Workspace: spec_verify_tree_workspace_size(B, N, V) bytes
 * (zeroed once, as for the other calls).
 */
size_t spec_verify_tree_workspace_size(int B, int N, int V);

int spec_verify_tree_greedy(const void *node_logits, int t_dtype, int64_t stride_b,
                            int64_t stride_node, const int32_t *parent, const int32_t *tokens,
                            int B, int N, int V, int32_t *accepted_len, int32_t *path,
                            int32_t *out_tokens, void *workspace, size_t workspace_bytes,
                            void *stream);

/*
 * Stochastic verify of a draft token tree (EAGLE-style tree drafting).
 *
 * "Accelerating Sonar through speculation", section "EAGLE": the tree holds
 * the Top-K candidates of every node; the longest acceptable path is kept
 * and the target adds one token.  The siblings are fixed candidates, so the
 * draft distribution behind each child is a point mass on its token, and
 * speculative rejection over the siblings in node order reads: at node u,
 * with p = softmax(row u / T), the residual mass R = 1 and the rejected set
 * E empty, child c (token x) is accepted iff x is in [0, V), x is not in E
 * and u_c * R < p(x); a rejected child puts x in E and takes p(x) off R.
 * The walk enters the accepted child; when none is accepted, the last token
 * is drawn from p restricted to the vocabulary outside E (Gumbel-max over
 * l/T).  The committed tokens follow the target's distribution at every
 * depth.  Draws (Philox4x32-10, key = seed, counter (c0, position,
 * seq_offset + b, tag)): u_c is the acceptance draw of position c - 1; the
 * final draw uses position u, tag CORRECTION when u has children and BONUS
 * at a leaf -- so a chain tree gives exactly spec_verify_stochastic with
 * one-hot draft distributions.
 *
 * node_logits, parent, tokens and the outputs are laid out as for
 * spec_verify_tree_greedy (out_tokens [B, N]: the n accepted tokens, the
 * drawn token, then -1).  temperature > 0 (normal, finite).  An invalid or
 * repeated sibling token is never accepted (SV_FLAG_INVALID_TOKEN for an
 * invalid one); a node with an invalid parent is never entered
 * (SV_FLAG_INVALID_TREE); if rounding leaves nothing outside E the draw
 * uses the whole row (SV_FLAG_RESIDUAL_FALLBACK).  1 <= N <= 64.
 * Workspace: spec_verify_tree_stochastic_workspace_size(B, N, V) bytes,
 * zeroed once as for the other calls (the call leaves it zeroed).  Three
 * kernel launches on `stream`.
 */
size_t spec_verify_tree_stochastic_workspace_size(int B, int N, int V);

int spec_verify_tree_stochastic(const void *node_logits, int t_dtype, int64_t stride_b,
                                int64_t stride_node, const int32_t *parent,
                                const int32_t *tokens, int B, int N, int V, float temperature,
                                uint64_t seed, uint32_t seq_offset, int32_t *accepted_len,
                                int32_t *path, int32_t *out_tokens, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * Device-side commit: the step after verify, with no host synchronisation.
 *
 * "Accelerating Sonar through speculation", section "Single-token MTP
 * scheduling": a small amount of extra GPU work spares the CPU-GPU sync after
 * acceptance -- the next tokens are written into place on the device, and
 * the host schedules the next step without waiting for the accepted lengths.
 *
 * For every sequence b, with n = accepted_len[b] (clamped to [0, k]) and
 * L = seq_len[b]: the n + 1 committed tokens out_tokens[b, 0..n] are written
 * to token_buf[b*buf_stride + L .. L+n]; seq_len[b] becomes L + n + 1; and
 * next_input[b] (nullable) receives out_tokens[b, n], the input of the next
 * decoding step (the position shift of an MTP draft is the caller's
 * indexing).  Tokens are copied as they are, -1 included.
 *
 * accepted_len [B], out_tokens [B, k+1] (as the verify calls write them),
 * seq_len [B] in/out, token_buf [B, >= capacity] (row stride buf_stride >=
 * capacity, in elements), next_input [B] or NULL: int32 device arrays.
 * Tokens that would land at or past `capacity` are dropped, seq_len stops at
 * capacity, and SV_FLAG_CAPACITY is set in `workspace` (a verify workspace,
 * nullable: then the flag is not reported).  A negative seq_len is read as 0.
 * One small launch on `stream`; B == 0 does nothing.
 */
int spec_verify_commit(const int32_t *accepted_len, const int32_t *out_tokens, int B, int k,
                       int32_t *seq_len, int32_t *token_buf, int64_t buf_stride, int capacity,
                       int32_t *next_input, void *workspace, void *stream);

/*
 * Philox4x32-10 (Salmon et al., SC'11) on the device, as the verify kernels
 * draw it: out[j] = Philox(counters[j], key = (seed lo, seed hi)).
 * counters and out are device arrays of n uint32x4 (16-byte aligned).
 */
int spec_verify_philox4x32_10(const uint32_t *counters, int64_t n, uint64_t seed,
                              uint32_t *out, void *stream);

/*
 * Greedy verify without any allocation.  The pages have no counterpart: this
 * is a library convenience for callers that cannot allocate device memory on
 * the verify path (an external allocator or pool owns the device, the call
 * runs in a real-time loop where an allocation may block or fail) and cannot
 * keep a workspace of their own.
 *
 * Same arguments, layouts and results as spec_verify_greedy, minus the
 * workspace: the library uses a fixed device array of
 * SV_NOALLOC_SCRATCH_BYTES that it carries in its image (every GPU that loads
 * the library holds it until the process exits).  Each call clears the part
 * it needs with cudaMemsetAsync on `stream` (all but the sticky status word),
 * then runs greedy verify on it; nothing is allocated or freed.
 *  - Returns SV_ERR_WORKSPACE when spec_verify_workspace_size(B, 1, k, V)
 *    exceeds SV_NOALLOC_SCRATCH_BYTES (at V = 128256: B <= 782 at k = 8,
 *    B <= 1448 at k = 4, B <= 208 at k = 32), SV_ERR_INVALID_ARG for sizes
 *    outside the limits, and otherwise what spec_verify_greedy returns.
 *  - Every call looks up the array's device address (cudaGetSymbolAddress,
 *    host-side, with the caller's device current); the first call on a device
 *    also loads the library's device code there, so make it before any
 *    stream capture.
 *  - All calls share the array: calls whose kernels may overlap on the GPU
 *    (unordered streams) race.  Order them on one stream.
 *  - Errors seen on the device (SV_FLAG_* bits: a draft token outside [0, V),
 *    a device wait that timed out) accumulate in the array's status word;
 *    read them with spec_verify_greedy_noalloc_read_device_status.
 */
#define SV_NOALLOC_SCRATCH_BYTES ((size_t)2 << 20)

int spec_verify_greedy_noalloc(const void *target_logits, int t_dtype, int64_t t_stride_b,
                               int64_t t_stride_pos, const int32_t *draft_tokens, int B, int k,
                               int V, int32_t *accepted_len, int32_t *out_tokens, void *stream);

/*
 * The sticky device status word (SV_FLAG_* bits) of spec_verify_greedy_noalloc
 * on the current device: copied into *flags_host (a host pointer) and, if
 * `clear` is nonzero, reset.  SYNCHRONISES `stream`; allocates nothing.  No
 * counterpart on the pages.
 */
int spec_verify_greedy_noalloc_read_device_status(uint32_t *flags_host, int clear,
                                                  void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SPEC_VERIFY_H */
