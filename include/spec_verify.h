/*
 * spec_verify.h -- C ABI of libspecverify, the verify/accept step of
 * speculative decoding on NVIDIA B200 (sm_100a).
 *
 * The method comes from three web pages, cited by title and section:
 *   [atlas]   "Speculative Decoding —— 无损加速自回归 decode" (llm-infra-atlas):
 *             §0 latency formula, §2 notation (p = target, q = draft, gamma,
 *             bonus token, correction / residual, tree attention).
 *   [kevins]  "Speculative Decoding：投机解码的真实收益、校正采样与生产边界"
 *             (ricardokevins notes): "draft / verify / accept" steps,
 *             "sampling correction" a(x) = min(1, p(x)/q(x)) and
 *             r(x) = max(p(x)-q(x),0) / sum_y max(p(y)-q(y),0).
 *   [origins] zdszero "spec_origins" page: "Blockwise Parallel Decoding"
 *             (verify = longest prefix equal to the argmax), "Speculative
 *             Decoding" (acceptance rules 1-3, why lossless, closed form),
 *             "SpecInfer" (token tree, ancestor-only mask), "In SGLang"
 *             (verify_tree_greedy, target-only tree sampling with prob_acc,
 *             threshold_single / threshold_acc, relu(target - draft_probs)).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument is DEVICE memory owned by the caller, except the
 *   host output of spec_read_device_status.  The library allocates nothing.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *   default stream).  Argument errors are detected on the host before any
 *   launch and returned synchronously; nothing is enqueued then.  A failed
 *   launch returns SPEC_ERR_CUDA.
 * - Per-sequence input errors found on the device (non-finite logits, an
 *   all -inf row, a token id outside [0, V), a temperature that is not a
 *   finite normal positive f32, a malformed parent array) never trap: the
 *   sequence gets out_num_accepted[b] = -1 and every output slot -1, and the
 *   bit (1 << SPEC_ERR_DEVICE_INPUT) is OR-ed into the workspace status word
 *   (read it with spec_read_device_status).
 * - Logit rows: row r of sequence b starts at element (b*R + r) * row_stride
 *   of its array (R = rows per sequence of that array).  Each row's first
 *   byte must be 16-byte aligned: base pointer 16-byte aligned and
 *   row_stride * element size a multiple of 16 bytes (a multiple of 8 bf16
 *   or 4 f32 elements).  row_stride >= V.
 * - Temperature softmax: p = softmax(logits / T) per row, computed in f32
 *   with f32 accumulation (fp64 across chunks); T is per sequence.
 * - Uniforms (coins, final_u) are caller-supplied f32 values in [0, 1).
 *   Every random choice of a call is a deterministic function of them: the
 *   same inputs give bit-identical outputs.  A coin of exactly 0 passes
 *   coin <= ratio even when the ratio is 0, i.e. it accepts a token the
 *   target gives probability 0; draw coins from (0, 1) to exclude that.
 * - Inverse-CDF draws scan the vocabulary in index order 0..V-1 and pick
 *   the smallest j with u * S < C_j (C = running sum of the weights, S the
 *   total): zero-weight tokens are never drawn.
 * - Workspace: caller-owned device scratch of spec_workspace_bytes() bytes,
 *   256-byte aligned, zero-filled once by spec_workspace_init() before first
 *   use and again whenever it is reused for another entry point or another
 *   batch size.  Its arrival counters reset themselves, so it can be reused
 *   by any number of calls of that shape, and captured in CUDA graphs, on
 *   ONE stream at a time (concurrent calls sharing a workspace race).
 * - Limits: 1 <= gamma <= SPEC_MAX_GAMMA, 1 <= N <= SPEC_MAX_NODES,
 *   0 <= max_depth <= SPEC_MAX_DEPTH, 1 <= V <= SPEC_MAX_V, B >= 0
 *   (B == 0 returns SPEC_OK and launches nothing).
 */
#ifndef SPEC_VERIFY_H
#define SPEC_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPEC_MAX_GAMMA 16
#define SPEC_MAX_NODES 256
#define SPEC_MAX_DEPTH 64
#define SPEC_MAX_V (1 << 20)

typedef enum {
    SPEC_OK = 0,
    SPEC_ERR_INVALID_ARG = 1,   /* host-side argument check failed; nothing launched */
    SPEC_ERR_UNSUPPORTED = 2,   /* valid but unsupported combination (e.g. no sm_100 device) */
    SPEC_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    SPEC_ERR_DEVICE_INPUT = 4,  /* (status bit) a sequence had invalid device-side inputs */
    SPEC_ERR_TIMEOUT = 5,       /* (status bit) a bounded device-side wait gave up */
    SPEC_ERR_WORKSPACE = 6,     /* workspace too small or misaligned */
    SPEC_ERR_COPY_IN_FLIGHT = 7 /* (status bit) after a timeout, the wait that lets a CTA's own bulk
                                   copy land gave up too: the copy may still have been writing that
                                   CTA's shared memory when it went on (results of the call are
                                   undefined) */
} spec_status;

typedef enum { SPEC_F32 = 0, SPEC_BF16 = 1 } spec_dtype;

typedef enum {
    SPEC_ENTRY_CHAIN = 0,
    SPEC_ENTRY_TREE_GREEDY = 1,
    SPEC_ENTRY_TREE_SAMPLE = 2,
    SPEC_ENTRY_TREE_MSS = 3
} spec_entry;

/*
 * spec_verify_chain -- chain speculative sampling, one round for B sequences.
 * [origins] "Speculative Decoding", acceptance rules 1-3; [kevins] "sampling
 * correction" a(x), r(x); the p/q rejection path that [origins] "In SGLang"
 * runs for chains (topk = 1).
 *
 * For each sequence b, with p_i = softmax(target row i / T_b), i in [0,gamma],
 * and q_i the draft distribution at position i:
 *   1. draft token x_i is accepted iff coins[b,i] <= p_i(x_i) / q_i(x_i)
 *      (ratio +inf when q_i(x_i) = 0), for i = 0, 1, ... until the first
 *      rejection k (k = gamma if none);
 *   2. if k < gamma the correction token is drawn with final_u[b] from
 *      norm(max(0, p_k - q_k)); if that mass is zero (rounding only) it is
 *      drawn from p_k;
 *   3. if k = gamma the bonus token is drawn with final_u[b] from p_gamma.
 *
 * target_logits  [B, gamma+1, t_row_stride] of tdt, read-only.
 * draft          [B, gamma, d_row_stride]: logits of ddt when draft_is_probs
 *                = 0 (q_i = softmax(draft row i / T_b), same T as the
 *                target), or f32 probabilities used as given when
 *                draft_is_probs = 1 (ddt must be SPEC_F32).  Read-only.
 * draft_tokens   [B, gamma] int32 in [0, V).
 * temperature    [B] f32.
 * coins          [B, gamma] f32, coins[b,i] is the uniform of position i.
 * final_u        [B] f32.
 * out_tokens     [B, gamma+1] int32: x_0..x_{k-1}, then the correction or
 *                bonus token at index k, then -1.
 * out_num_accepted [B] int32: k in [0, gamma], or -1 (invalid sequence).
 * diag           nullable, [B, 2*gamma+1] f32: p_i(x_i) for i < gamma,
 *                then q_i(x_i) for i < gamma, then S = the mass of the
 *                distribution the last token was drawn from before
 *                normalisation (sum_j max(0, p_k(j) - q_k(j)) on a
 *                rejection, 1 for a bonus).
 * workspace      >= spec_workspace_bytes(SPEC_ENTRY_CHAIN, B, gamma, V).
 */
spec_status spec_verify_chain(int B, int gamma, int V,
                              const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                              const void* draft, spec_dtype ddt, int draft_is_probs,
                              int64_t d_row_stride,
                              const int32_t* draft_tokens, const float* temperature,
                              const float* coins, const float* final_u,
                              int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * spec_verify_chain_filtered -- spec_verify_chain under top-k / top-p
 * filtered temperature sampling.  [kevins] "draft / verify / accept" (real
 * serving samples with temperature, top-p and top-k, and verify must stay
 * unbiased under them) and "production limits" (a wider top-p lowers
 * acceptance); the pages do not define the filters, so the textbook ones:
 *   p'_i = softmax(target row i / T_b) restricted to the kept tokens and
 *   renormalised, where the kept tokens are: top-k (0 < top_k[b] < V) the
 *   tokens whose logit is >= the top_k-th largest logit (ties kept); then
 *   top-p (0 < top_p[b] < 1) the smallest set of whole groups of equal
 *   logits, from the largest down, whose share of the top-k set's mass
 *   reaches top_p[b].
 * Draft logits are filtered the same way (the drafter sampled from its own
 * filtered distribution); draft probabilities are used as given.  Rules 1-3
 * then run on p' and q' exactly as in spec_verify_chain, so the emitted
 * tokens follow the filtered target distribution.
 *
 * Arguments as spec_verify_chain, plus:
 * top_k          [B] int32, nullable (NULL or 0 = no top-k); < 0 makes the
 *                sequence invalid.
 * top_p          [B] f32, nullable (NULL or 1 = no top-p); outside (0, 1]
 *                makes the sequence invalid.  At least one of the two must
 *                be non-NULL.
 * diag           p'_i(x_i), q'_i(x_i), then the final mass S as in
 *                spec_verify_chain.
 * workspace      >= spec_workspace_bytes(SPEC_ENTRY_CHAIN, B, gamma, V).
 * Cost: per filtered row, one CTA walks the row 2-4 times (bf16; 4-8 for f32)
 * to find its thresholds by radix descent (16-bit / 32-bit order keys, 8 bits
 * per pass; counts for top-k, fixed-point masses in 2^-40 units for top-p),
 * and the correction or bonus is drawn over the whole filtered row.
 */
spec_status spec_verify_chain_filtered(int B, int gamma, int V,
                                       const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                       const void* draft, spec_dtype ddt, int draft_is_probs,
                                       int64_t d_row_stride,
                                       const int32_t* draft_tokens, const float* temperature,
                                       const float* coins, const float* final_u,
                                       const int32_t* top_k, const float* top_p,
                                       int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * spec_verify_chain_filtered_lazy -- spec_verify_chain_filtered as a
 * row-on-demand level walk (the lazy conventions below): per position the
 * statistics and filter records of only the rows the still-active sequences
 * reach (target row i, draft-logit row i; row gamma after a full acceptance),
 * then one decision per active sequence; then the draw.  Same arguments,
 * workspace size and outputs; rows never read are not validated and the
 * diagnostics hold NaN where nothing was evaluated.
 */
spec_status spec_verify_chain_filtered_lazy(int B, int gamma, int V,
                                       const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                       const void* draft, spec_dtype ddt, int draft_is_probs,
                                       int64_t d_row_stride,
                                       const int32_t* draft_tokens, const float* temperature,
                                       const float* coins, const float* final_u,
                                       const int32_t* top_k, const float* top_p,
                                       int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * spec_verify_tree_greedy -- greedy verify of a draft token tree.
 * [origins] "In SGLang" (greedy goes through verify_tree_greedy) and
 * "Blockwise Parallel Decoding" (verify keeps the longest prefix equal to
 * the scoring model's own argmax, so the output equals greedy decoding);
 * [origins] "SpecInfer" (tree flattened, ancestors before descendants).
 *
 * g_n = argmax_j target[b, n, j] (lowest index among equal maxima; a NaN
 * anywhere in the sequence's rows makes it invalid).  Walk: cur = 0; the
 * first child c of cur in increasing node index with tokens[b,c] == g_cur is
 * accepted and becomes cur; stop when no child matches.  Emitted: the
 * accepted draft tokens, then the bonus g_cur.
 *
 * target_logits  [B, N, t_row_stride]; row n holds the target logits at tree
 *                node n (node 0 = the last verified token, the root).
 * tokens         [B, N] int32; tokens[b,0] is not read; others in [0, V).
 * parents        [B, N] int32; parents[b,0] = -1; 0 <= parents[b,n] < n; every
 *                node's depth (root = 0) <= max_depth.
 * out_accept_index [B, max_depth+1] int32: node ids of the accepted path,
 *                root first (k+1 entries), then -1.
 * out_tokens     [B, max_depth+1] int32: the k accepted draft tokens, the
 *                bonus token at index k, then -1.
 * out_num_accepted [B] int32: k, or -1.
 * workspace      >= spec_workspace_bytes(SPEC_ENTRY_TREE_GREEDY, B, N, V).
 * Temperature plays no part.
 */
spec_status spec_verify_tree_greedy(int B, int N, int V, int max_depth,
                                    const void* target_logits, spec_dtype tdt,
                                    int64_t t_row_stride,
                                    const int32_t* tokens, const int32_t* parents,
                                    int32_t* out_accept_index, int32_t* out_tokens,
                                    int32_t* out_num_accepted,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * spec_verify_tree_sample -- target-only tree sampling.
 * [origins] "In SGLang": tree_speculative_sampling_target_only, a SpecInfer
 * style walk down the tree that tries the next sibling after a rejection;
 * draft probabilities are zeros and acceptance reads the target only.
 *
 * p_n = softmax(target row n / T_b).  cur = 0.  At cur the children c_1..c_m
 * (increasing node index) are tried in order with prob_acc += p_cur(tok_c):
 * c is accepted iff coins[b,cur] <= prob_acc / threshold_acc or
 * p_cur(tok_c) >= threshold_single; on acceptance cur = c and the walk goes
 * one level down (with coins[b,c]); a child that is not accepted is
 * rejected.  The walk stops when no child of cur is accepted or cur has no
 * children.  The last token is drawn with final_u[b] from
 * relu(p_cur - d_cur), where d_cur is the draft_probs row of cur (zeros when
 * draft_probs is NULL) with the entries of cur's rejected children replaced
 * by their target probabilities.  draft_probs is never written: the
 * replacement is kept on chip.  With both thresholds 1 the emitted tokens
 * are distributed exactly as the target's.
 *
 * Arguments as spec_verify_tree_greedy, plus:
 * temperature    [B] f32.
 * coins          [B, N] f32: coins[b,n] is the uniform used while visiting n.
 * final_u        [B] f32.
 * draft_probs    nullable, [B, N, dp_row_stride] f32.
 * threshold_single, threshold_acc  host f32, > 0 (1.0 = lossless).
 * diag           nullable, [B, N+1] f32: p_parent(n)(tokens[b,n]) for n >= 1
 *                (0 at n = 0), then S = the mass of relu(p_cur - d_cur).
 * workspace      >= spec_workspace_bytes(SPEC_ENTRY_TREE_SAMPLE, B, N, V).
 */
spec_status spec_verify_tree_sample(int B, int N, int V, int max_depth,
                                    const void* target_logits, spec_dtype tdt,
                                    int64_t t_row_stride,
                                    const int32_t* tokens, const int32_t* parents,
                                    const float* temperature, const float* coins,
                                    const float* final_u,
                                    const float* draft_probs, int64_t dp_row_stride,
                                    float threshold_single, float threshold_acc,
                                    int32_t* out_accept_index, int32_t* out_tokens,
                                    int32_t* out_num_accepted, float* diag,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * spec_verify_tree_sample_filtered -- target-only tree sampling under
 * top-k / top-p filtered temperature sampling ([kevins] "draft / verify /
 * accept": serving samples with temperature, top-k and top-p).  Every
 * node's target row is filtered as spec_verify_chain_filtered filters a
 * target row (top-k with ties kept, then top-p over whole groups of equal
 * logits, renormalised), per sequence; the walk, prob_acc, the thresholds
 * and the final relu(p'_cur - d_cur) then use the filtered distributions.
 * draft_probs rows are used as given.  With both thresholds 1 the emitted
 * tokens are distributed exactly as the filtered target's.
 *
 * Arguments as spec_verify_tree_sample, plus top_k [B] int32 and top_p [B]
 * f32 as in spec_verify_chain_filtered (each nullable, not both; top_k < 0 or
 * top_p outside (0, 1] makes that sequence invalid).  diag as
 * spec_verify_tree_sample, with the filtered probabilities.  Same workspace
 * as spec_verify_tree_sample.  Three launches: the statistics, the filter
 * (one CTA of 1024 threads per node row, about 192 KB of shared memory for
 * bf16 rows), the walk.
 */
spec_status spec_verify_tree_sample_filtered(int B, int N, int V, int max_depth,
                                             const void* target_logits, spec_dtype tdt,
                                             int64_t t_row_stride,
                                             const int32_t* tokens, const int32_t* parents,
                                             const float* temperature, const float* coins,
                                             const float* final_u,
                                             const float* draft_probs, int64_t dp_row_stride,
                                             float threshold_single, float threshold_acc,
                                             const int32_t* top_k, const float* top_p,
                                             int32_t* out_accept_index, int32_t* out_tokens,
                                             int32_t* out_num_accepted, float* diag,
                                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * spec_verify_tree_sample_filtered_lazy -- the same results, filtering only
 * the rows the walk reaches: per level the statistics and the filter record
 * of each active sequence's current node, then the decisions (three
 * dependent launches per level), then the draw.  Differences as the other
 * _lazy entry points: diag holds NaN for the children of unvisited nodes,
 * and rows that are never read are not validated.
 */
spec_status spec_verify_tree_sample_filtered_lazy(int B, int N, int V, int max_depth,
                                                  const void* target_logits, spec_dtype tdt,
                                                  int64_t t_row_stride,
                                                  const int32_t* tokens, const int32_t* parents,
                                                  const float* temperature, const float* coins,
                                                  const float* final_u,
                                                  const float* draft_probs, int64_t dp_row_stride,
                                                  float threshold_single, float threshold_acc,
                                                  const int32_t* top_k, const float* top_p,
                                                  int32_t* out_accept_index, int32_t* out_tokens,
                                                  int32_t* out_num_accepted, float* diag,
                                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * spec_verify_tree_mss -- tree verification with a draft distribution
 * (multi-step speculative sampling).  [origins] "SpecInfer", MSS bullet:
 * after a child is rejected the target distribution is replaced by the
 * residual norm(max(0, p - q)) and the next sibling is tried; the emitted
 * tokens keep the target distribution when the children of every node were
 * drawn independently from that node's draft distribution.
 *
 * p = softmax(target row cur / T_b) and q = draft_probs row cur, starting at
 * the root.  The children of cur are tested in increasing node index: child
 * c is accepted iff coins[b,c] <= p(tokens[b,c]) / q(tokens[b,c]) (ratio +inf
 * when q = 0); on acceptance the walk moves to c (fresh p and q of c); on
 * rejection p <- max(0, p - q) / S, S = sum_j max(0, p_j - q_j) (p is kept
 * when S is not positive: rounding only), and the next sibling is tried.
 * When no child of cur is accepted, or cur is a leaf, the last token is
 * drawn with final_u[b] from the current p.
 *
 * Arguments as spec_verify_tree_greedy, plus:
 * temperature    [B] f32.
 * coins          [B, N] f32: coins[b,c] is the uniform of the test of child
 *                c (coins[b,0] is not read).  Note the difference from
 *                spec_verify_tree_sample, whose coins belong to the visited
 *                parent.
 * final_u        [B] f32.
 * draft_probs    [B, N, dp_row_stride] f32, required: row n is the draft
 *                distribution from which the children of node n were drawn.
 *                Only the rows of visited nodes are read; the drafted
 *                tokens' entries must be finite and >= 0 (else the sequence
 *                is invalid).  Never written.
 * diag           nullable, [B, N+1] f32: p(tokens[b,c]) at the test of child
 *                c (NaN for children never tested, and at n = 0), then the
 *                last residual mass S at the final node (1 without one).
 * workspace      >= spec_workspace_bytes(SPEC_ENTRY_TREE_MSS, B, N, V).
 * Each rejection costs one extra pass over the (target, q) row pair of the
 * node.
 *
 * spec_verify_tree_mss_lazy: the same call, walking level by level and
 * reading only the rows of the visited nodes (see the lazy variants below):
 * outputs bit-identical for valid inputs; rows never read are not validated.
 */
spec_status spec_verify_tree_mss(int B, int N, int V, int max_depth,
                                 const void* target_logits, spec_dtype tdt,
                                 int64_t t_row_stride,
                                 const int32_t* tokens, const int32_t* parents,
                                 const float* temperature, const float* coins,
                                 const float* final_u,
                                 const float* draft_probs, int64_t dp_row_stride,
                                 int32_t* out_accept_index, int32_t* out_tokens,
                                 int32_t* out_num_accepted, float* diag,
                                 void* workspace, size_t workspace_bytes, void* stream);
spec_status spec_verify_tree_mss_lazy(int B, int N, int V, int max_depth,
                                      const void* target_logits, spec_dtype tdt,
                                      int64_t t_row_stride,
                                      const int32_t* tokens, const int32_t* parents,
                                      const float* temperature, const float* coins,
                                      const float* final_u,
                                      const float* draft_probs, int64_t dp_row_stride,
                                      int32_t* out_accept_index, int32_t* out_tokens,
                                      int32_t* out_num_accepted, float* diag,
                                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * spec_verify_chain_noalloc -- spec_verify_chain without a caller workspace.
 * The pages have no counterpart of this entry point; it exists for callers
 * that cannot allocate device memory where they verify: a plugin running
 * inside an engine whose allocator owns all GPU memory, a decode loop that
 * cannot afford the implicit device synchronisation of cudaMalloc/cudaFree,
 * or a host thread without access to an allocator.  It allocates nothing and
 * calls no allocating routine.
 *
 * Arguments, semantics, outputs and error behaviour are those of
 * spec_verify_chain, minus workspace and workspace_bytes.  The scratch is a
 * built-in device array of SPEC_NOALLOC_SCRATCH_BYTES (16 MiB) that every GPU
 * loading the library holds until the process exits.  A shape whose scratch
 * need (spec_workspace_bytes(SPEC_ENTRY_CHAIN, B, gamma, V)) exceeds it is
 * rejected with SPEC_ERR_WORKSPACE before anything is enqueued.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture.
 * - All calls share the one array, which keeps the previous call's contents;
 *   each call first clears (cudaMemsetAsync on `stream`) the parts that must
 *   start at zero.  Calls whose executions overlap on the GPU -- on different
 *   streams, or from different host threads -- race on the array and give
 *   undefined results: serialise them.
 * - Device-side input errors are reported through out_num_accepted = -1; the
 *   status word lives in the shared array and is not readable by the caller.
 */
#define SPEC_NOALLOC_SCRATCH_BYTES (16u << 20)
spec_status spec_verify_chain_noalloc(int B, int gamma, int V,
                                      const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                      const void* draft, spec_dtype ddt, int draft_is_probs,
                                      int64_t d_row_stride,
                                      const int32_t* draft_tokens, const float* temperature,
                                      const float* coins, const float* final_u,
                                      int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                                      void* stream);

/*
 * Lazy (row-on-demand) variants: spec_verify_chain_lazy,
 * spec_verify_tree_greedy_lazy, spec_verify_tree_sample_lazy.
 * [origins] "Speculative Decoding" (rules 1-3 look at position i only after
 * positions 0..i-1 were accepted) and "SpecInfer" / "In SGLang" (the tree
 * walk only ever reads the rows of the nodes it visits); [atlas] §0 (verify
 * time is a cost the round pays whatever is accepted).
 *
 * Same arguments, workspace size (same `entry` as the dense function),
 * outputs and error reporting as the function without the suffix; for valid
 * inputs out_tokens, out_num_accepted and out_accept_index are bit-identical
 * to it.  Instead of reading every row, they walk level by level on the
 * device -- the rows the still-active sequences need, then one decision per
 * active sequence -- and read about (accepted tokens + 1) rows (chain: row
 * pairs) per sequence.  Costs and differences:
 * - 2 kernel launches per level (gamma+1 levels for the chain, max_depth+1
 *   for trees, launched whether or not a sequence is still active) plus the
 *   final draw: worth it when rows are large and rejections come early.
 * - Rows that are never read are not validated: a non-finite logit in a row
 *   past the stopping point, or an invalid drafted token past the first
 *   rejection, does not make the sequence invalid.  Tree structure and
 *   temperature are always validated.
 * - diag: only evaluated entries are written; the rest hold NaN (chain:
 *   positions after the first rejection; tree sampling: children of nodes
 *   the walk did not visit).  Evaluated entries equal the dense ones.
 */
spec_status spec_verify_chain_lazy(int B, int gamma, int V,
                                   const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                   const void* draft, spec_dtype ddt, int draft_is_probs,
                                   int64_t d_row_stride,
                                   const int32_t* draft_tokens, const float* temperature,
                                   const float* coins, const float* final_u,
                                   int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                                   void* workspace, size_t workspace_bytes, void* stream);
spec_status spec_verify_tree_greedy_lazy(int B, int N, int V, int max_depth,
                                         const void* target_logits, spec_dtype tdt,
                                         int64_t t_row_stride,
                                         const int32_t* tokens, const int32_t* parents,
                                         int32_t* out_accept_index, int32_t* out_tokens,
                                         int32_t* out_num_accepted,
                                         void* workspace, size_t workspace_bytes, void* stream);
spec_status spec_verify_tree_sample_lazy(int B, int N, int V, int max_depth,
                                         const void* target_logits, spec_dtype tdt,
                                         int64_t t_row_stride,
                                         const int32_t* tokens, const int32_t* parents,
                                         const float* temperature, const float* coins,
                                         const float* final_u,
                                         const float* draft_probs, int64_t dp_row_stride,
                                         float threshold_single, float threshold_acc,
                                         int32_t* out_accept_index, int32_t* out_tokens,
                                         int32_t* out_num_accepted, float* diag,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Vocabulary-parallel chain verify: the target (and draft) logits of every
 * row are sharded along the vocabulary over the `world` ranks of a tensor-
 * parallel group; rank r holds columns [vocab_offset_r, vocab_offset_r +
 * V_shard_r) and the shards tile [0, V).  The pages assume one device holds
 * whole rows ([origins] "Speculative Decoding" rules 1-3); these calls split
 * the same rules into per-shard steps joined by three small exchanges that
 * the caller performs (NCCL all-gather / all-reduce), giving the tokens and
 * counts of spec_verify_chain up to rounding (shard sums are combined in
 * rank order):
 *   1. spec_vp_chain_stats on every rank -> rec_out [B, 2*gamma+1] records of
 *      spec_vp_record_bytes() bytes; all-gather into rec_all [world, B, ...]
 *      in rank order;
 *   2. spec_vp_chain_decide on every rank (identical results): accepted
 *      tokens, out_num_accepted, p/q diagnostics, and the per-sequence state
 *      the next steps read from the workspace;
 *   3. spec_vp_chain_residual -> mass_out [B] f64, the shard's part of the
 *      mass of the last token's distribution (its chunk masses stay in the
 *      workspace for step 4); all-gather into mass_all [world, B];
 *   4. spec_vp_chain_sample -> tok_out [B] int32: the global token id on the
 *      rank whose shard holds u*S, -1 elsewhere; all-reduce MAX;
 *   5. spec_vp_chain_finish writes the reduced token at position k of
 *      out_tokens.
 * Each rank uses one workspace of spec_workspace_bytes(SPEC_ENTRY_CHAIN, B,
 * gamma, V_shard) for all five steps of a round (V_shard of that rank).
 * Argument conventions otherwise as spec_verify_chain (rows of the shard,
 * strides in elements); draft_tokens are global ids in [0, V).
 */
size_t spec_vp_record_bytes(void);
spec_status spec_vp_chain_stats(int B, int gamma, int V_shard, int vocab_offset,
                                const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                const void* draft, spec_dtype ddt, int draft_is_probs, int64_t d_row_stride,
                                const int32_t* draft_tokens, const float* temperature, void* rec_out,
                                void* workspace, size_t workspace_bytes, void* stream);
spec_status spec_vp_chain_decide(int B, int gamma, int V, int V_shard, int world, const void* rec_all,
                                 int draft_is_probs,
                                 const int32_t* draft_tokens, const float* temperature, const float* coins,
                                 int32_t* out_tokens, int32_t* out_num_accepted, float* diag,
                                 void* workspace, size_t workspace_bytes, void* stream);
spec_status spec_vp_chain_residual(int B, int gamma, int V_shard, int world, int rank,
                                   const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                   const void* draft, spec_dtype ddt, int draft_is_probs, int64_t d_row_stride,
                                   const void* rec_all, double* mass_out,
                                   void* workspace, size_t workspace_bytes, void* stream);
spec_status spec_vp_chain_sample(int B, int gamma, int V_shard, int vocab_offset, int world, int rank,
                                 const void* target_logits, spec_dtype tdt, int64_t t_row_stride,
                                 const void* draft, spec_dtype ddt, int draft_is_probs, int64_t d_row_stride,
                                 const float* final_u, const void* rec_all, const double* mass_all,
                                 int32_t* tok_out, float* diag,
                                 void* workspace, size_t workspace_bytes, void* stream);
spec_status spec_vp_chain_finish(int B, int gamma, int V_shard, const int32_t* tok, int32_t* out_tokens,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * spec_workspace_bytes -- workspace size for one entry point and shape.
 * rows = gamma for SPEC_ENTRY_CHAIN (sized for draft logits, which also
 * covers draft probabilities), N for the tree entry points.  Returns 0 for
 * out-of-range arguments.  Pure host function.
 */
size_t spec_workspace_bytes(int entry, int B, int rows, int V);

/* spec_workspace_init -- zero-fill `bytes` of the workspace on `stream`. */
spec_status spec_workspace_init(void* workspace, size_t bytes, void* stream);

/*
 * spec_read_device_status -- copy the workspace status word to *status_out
 * (a bit mask: bit c set <=> status code c occurred since the last read),
 * then clear it.  Synchronises `stream`.
 */
spec_status spec_read_device_status(void* workspace, int* status_out, void* stream);

/*
 * spec_profile_events -- kernel timing hook.  While set (non-NULL), every
 * later verify call on this host thread records `start_event` on its stream
 * just before launching its row-statistics kernel (the kernel that streams
 * every logit row, which dominates each call) and `stop_event` just after it,
 * so cudaEventElapsedTime gives that kernel's duration (for the lazy
 * variants: the whole level walk and final draw).  Both are
 * cudaEvent_t handles owned by the caller; NULL, NULL switches the hook off.
 * Inside stream capture the records become external event nodes.
 */
spec_status spec_profile_events(void* start_event, void* stop_event);

/*
 * spec_debug_wait_budget -- testing hook for the device-side timeout path.
 * The finalize kernels stage data in shared memory with bulk copies and wait
 * for each copy with a bounded poll (by default 2^24 polls and 1 s); when the
 * first wait gives up they OR (1 << SPEC_ERR_TIMEOUT) into the status word,
 * wait again with the full budget so that the copy lands before the CTA goes
 * on (else also (1 << SPEC_ERR_COPY_IN_FLIGHT)), and then read the staged
 * statistics from global memory instead, or give up on the sequence (-1 in
 * its outputs) when the staged row pair was lost.  tries = 0 makes every first
 * wait give up at once while the copies land normally, which drives that
 * path without making any copy late; tries < 0 restores the default.
 * Applies to later calls on the calling host thread.  Not for production use.
 */
spec_status spec_debug_wait_budget(long long tries);

/*
 * spec_debug_filter_path -- testing hook for the top-k / top-p filters of bf16
 * rows.  Each filtered row is first resolved from its candidates: the values
 * within a factor 2^D of the row's largest probability (D = 12 in the filter
 * kernel, 14 in the on-demand and lazy walks, less with top-p alone when the
 * row's mass bound allows), counted per value in one pass into a window of
 * per-key counters fixed by the row statistics, and again with D + 6, then
 * D + 12, when a cut holds too few values or too little mass.  A row whose
 * candidates cannot hold the answer, or whose window would overflow the
 * kernel's shared memory, is resolved by a whole-row path (the 65536-key
 * value histogram in 1024-thread filter CTAs, else the windowed filter).
 * Both give the same record.
 * mode 0: the default paths, counting rows by path; mode 1: whole-row paths
 * only, counting; mode -1: the default paths, no counting (the state at load).
 * rows, if not NULL, receives three counts since the last read on the
 * current device -- [0] rows the candidates resolved at the first cut, [1]
 * rows left to a whole-row path, [2] rows the candidates resolved at a
 * deeper cut -- and resets them (a synchronous device read).  Applies to later calls
 * on the calling host thread.  Not for production use.
 */
spec_status spec_debug_filter_path(int mode, unsigned long long* rows);

/*
 * spec_launch_count -- number of kernels this library has launched (or, inside
 * stream capture, added to a graph) from the calling host thread since the
 * process started.  The difference across a call is that call's launch count.
 */
unsigned long long spec_launch_count(void);

/*
 * spec_debug_bounds_hits -- in a library compiled with -DSPEC_DEBUG_BOUNDS
 * (libspecverify_debug.so), every data-driven index the kernels use -- a
 * gathered token id, a parent link, a drawn chunk -- is range-checked on the
 * device; a failed check is counted and the access skipped (a token gathered
 * out of range reads as NaN, which invalidates its sequence).  This call
 * synchronises the device, stores the count since the last call in *hits and
 * clears it.  A library built without the flag returns SPEC_ERR_UNSUPPORTED
 * (and *hits = 0).  The checks cost time; they are for debugging.
 */
spec_status spec_debug_bounds_hits(unsigned long long* hits);

/* spec_status_string -- static description of a status code. */
const char* spec_status_string(spec_status status);

/* spec_last_error_detail -- detail of the last SPEC_ERR_INVALID_ARG /
 * SPEC_ERR_CUDA / SPEC_ERR_WORKSPACE returned on the calling host thread. */
const char* spec_last_error_detail(void);

#ifdef __cplusplus
}
#endif

#endif /* SPEC_VERIFY_H */
