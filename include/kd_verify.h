/*
 * kd_verify.h -- C ABI of libkdverify.so, the B200 (sm_100a) tree-verify step of
 * DDTree speculative decoding for Multi-head Latent Attention (MLA) models.
 *
 * One verify step (sources are the pages' titles and sections):
 *   0. kd_tree_build         the draft tree itself, best first from the drafter's
 *                            per-depth candidates ("The Architecture of Pragmatic
 *                            Ambition", "The Knowledge Architecture");
 *   1. kd_kv_write_nodes     the budget+1 node latents go to the next free slots,
 *                            root first ("The Architectural Keystone: Writing the
 *                            Model Header ...", "The Reasoning That Preceded the
 *                            Header");
 *   2. kd_tree_build_mask    per-node ancestor bitmasks from the parent array
 *                            ("The Architecture of Pragmatic Ambition", "The
 *                            Knowledge Architecture": attention over the tree with
 *                            a visibility mask);
 *   3. kd_tree_verify_attn   MLA attention in absorb form ("The Architecture of
 *                            Pragmatic Ambition", "The Thinking Process") of every
 *                            node and head over the committed cache and the node's
 *                            tree ancestors;
 *   4. kd_tree_accept        greedy walk to the longest path matching the target
 *                            argmax ("The Knowledge Architecture");
 *      kd_tree_accept_logits the same walk fed by the argmax of the target's
 *                            logits, both in one launch ("The Output Knowledge:
 *                            What This Message Creates");
 *   5. kd_kv_compact         the accepted path's latents, root included, gathered
 *                            into contiguous slots and the length advanced
 *                            ("The Reasoning That Preceded the Header"; read-all-
 *                            then-write, "Mistakes and Iterative Refinement").
 *
 * Conventions shared by every call
 *   - All pointers except those documented as host pointers are DEVICE pointers on
 *     the current CUDA device.  The caller allocates and owns every buffer,
 *     workspace included; the library allocates nothing and keeps no state besides
 *     cached device/function attributes.
 *   - Every call is asynchronous on `stream`; results are valid after the stream
 *     is synchronised.
 *   - bf16 tensors are passed as kd_bf16_t (the 16-bit pattern of a bfloat16).
 *   - Fixed MLA widths: latent d_c = 512, rope d_r = 64.  Limits: 1 <= n <= 128
 *     tree nodes (budget <= 127), 1 <= H <= 128 heads, B >= 1.
 *   - Request b's cache rows are c_kv[b*cap + j] (row stride kv_row_stride_c
 *     elements) and k_rope[b*cap + j] (row stride kv_row_stride_r elements); a
 *     576-wide interleaved layout is expressed by pointing k_rope at column 512
 *     and passing stride 576 for both.
 *   - Return value: KD_OK (0) or a negative KD_E* code.  Host-side validation
 *     happens before anything is enqueued; a failing call enqueues nothing.
 *   - Device-detected input errors (bad parent, cache overflow, bad accepted
 *     length, ...) never trap: the kernel ORs a KD_DEV_* bit into the caller's
 *     int32 device error word and treats the affected request as a no-op.  Read
 *     it with kd_read_device_error().  For kd_tree_verify_attn the error word is
 *     the first int32 of the workspace; the other calls take it as `dev_error`
 *     (may be NULL, in which case device errors are only skipped).
 */
#ifndef KD_VERIFY_H
#define KD_VERIFY_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t kd_bf16_t;

/* return codes */
#define KD_OK            0
#define KD_EINVAL       -1   /* null pointer, bad shape/limit, misaligned pointer or stride */
#define KD_ERANGE       -2   /* workspace too small / size beyond a documented maximum     */
#define KD_ELAUNCH      -3   /* a CUDA call failed; kd_strerror() gives the CUDA text       */
#define KD_ENODEV       -4   /* current device is not sm_100 (B200-class)                   */

/* device error bits (ORed into the device error word) */
#define KD_DEV_BAD_PARENT    0x01  /* parent[0] != -1 or parent[i] not in [0, i)       */
#define KD_DEV_CACHE_FULL    0x02  /* cache_len + n (or + len) exceeds cap, or < 0     */
#define KD_DEV_BAD_PATH      0x04  /* len not in [1, n] or path entry not in [0, n)     */
#define KD_DEV_BAD_POSITION  0x08  /* positions[b][i] != cache_len[b] + depth(i)       */
#define KD_DEV_TIMEOUT       0x10  /* a bounded wait inside a kernel gave up            */
#define KD_DEV_BAD_MASK      0x20  /* a node's mask lacks bit 0 (root) or its own bit   */
#define KD_DEV_BAD_PAGE      0x40  /* a paged cache's page id is outside the page pool  */

#define KD_D_C 512
#define KD_D_R 64
#define KD_MAX_NODES 128
#define KD_MAX_HEADS 128

/*
 * kd_tree_build_mask -- ancestor bitmasks and depths of B trees.
 *   parents [B][n] int32  topological: parents[b][0] == -1, 0 <= parents[b][i] < i.
 *   vis     [B][n][W] uint32 out, W = (n+31)/32: bit k of word k/32 of row i is set
 *           iff node k is node i or one of its ancestors.
 *   depth   [B][n] int32 out (may be NULL): edges from the root.
 *   A request with a bad parent array gets KD_DEV_BAD_PARENT and all-zero rows.
 */
int kd_tree_build_mask(const int32_t* parents, int B, int n, uint32_t* vis,
                       int32_t* depth, int32_t* dev_error, cudaStream_t stream);

/*
 * kd_verify_workspace_bytes -- workspace size for kd_tree_verify_attn with the
 * same B, n, H, cap and kv_splits.  Returns 0 for an invalid shape.
 *   - kv_splits = 0 sizes the split count the call itself would choose on the
 *     CURRENT device: the automatic policy depends on how many 2-CTA clusters of
 *     the attention kernel fit on it at once, which this function queries (and
 *     caches per device).  With no usable device (a build host) it assumes 74
 *     clusters, the B200 figure.  A workspace sized this way on the device that
 *     runs the call gives the call exactly that split count; on a device that
 *     would choose more splits the call lowers its choice to fit (see ws_bytes).
 *   - Layout (bytes): a 256-byte control block -- int32 device error word at 0;
 *     the first bounded wait that gave up at 4 and each warp's at 32..127 (bit 31
 *     set, CTA rank << 24, warp << 16, barrier << 4, parity); the scheduler's two
 *     uint64 counters at 8 and 16 -- then, with more than one split, the per-M-tile
 *     tickets [B * ceil(n H / 128)][2] int32, the partial lse [S][B n H] fp32 and
 *     the partial outputs [S][B n H][512] fp32, each region 256-byte aligned.
 *   - The workspace must be 256-byte aligned and start zeroed (e.g. from
 *     cudaMemset).  Every launch returns the counters and tickets to zero, so one
 *     workspace serves any number of calls in stream order; the error word is only
 *     ORed into (the caller clears it, e.g. with kd_read_device_error).  After a
 *     KD_DEV_TIMEOUT the kernel may have stopped mid-way: zero the whole control
 *     block and the tickets again before the next call.
 */
size_t kd_verify_workspace_bytes(int B, int n, int H, int64_t cap, int kv_splits);

/*
 * kd_tree_verify_attn -- masked MLA-absorb attention of every tree node over its
 * request's committed cache and its tree ancestors.
 *
 * For request b with L = cache_lens[b], node i, head h:
 *   V(i)  = {0 .. L-1}  U  {L + k : bit k of vis[b][i] set}        (node k at slot L+k)
 *   s_j   = scale * (q_nope_absorbed[b][i][h] . c_kv[j] + q_rope[b][i][h] . k_rope[j])
 *   out[b][i][h] = sum_{j in V(i)} softmax(s)_j * c_kv[j]          (512-wide latent)
 *   lse[b][i][h] = ln sum_{j in V(i)} exp(s_j)
 *
 *   q_nope_absorbed [B][n][H][512] bf16, contiguous (q_nope already multiplied by W_UK).
 *   q_rope          [B][n][H][64]  bf16, contiguous, already rotated.
 *   c_kv, k_rope    cache rows as described above, already holding the n node
 *                   latents at slots L..L+n-1; rotated keys.  Base pointers and
 *                   row strides must be 16-byte aligned (strides multiple of 8).
 *   cap             slots per request; requires cache_lens[b] + n <= cap.
 *   cache_lens [B]  int32 committed lengths (device).
 *   vis [B][n][W]   uint32 node masks (e.g. from kd_tree_build_mask).
 *   positions [B][n] int32 or NULL.  q_rope/k_rope arrive rotated, so positions do
 *                   not enter the arithmetic; when given they are checked against
 *                   cache_lens[b] + depth(i) and a mismatch sets KD_DEV_BAD_POSITION.
 *   scale           softmax scale applied to the raw dot products.
 *   out [B][n][H][512] bf16 out; lse [B][n][H] fp32 out (natural log; -inf if a
 *                   node sees no key, which cannot happen with a valid mask).
 *   workspace       >= kd_verify_workspace_bytes(B, n, H, cap, kv_splits) bytes
 *                   (ws_bytes, the caller's size), layout and lifetime as above.
 *   kv_splits       0 = automatic: the policy's split count, lowered until its
 *                   partials fit ws_bytes; otherwise the number of key-range
 *                   partitions per request (1 .. 64), combined by a log-sum-exp
 *                   merge inside the same launch.  An explicit count whose
 *                   workspace exceeds ws_bytes returns KD_ERANGE (nothing enqueued).
 *   out/lse must not alias any input.
 *   The work is one persistent launch of at most one 2-CTA cluster per SM pair;
 *   units (request, 128-row M tile, key partition) are handed out longest request
 *   first.  Every internal wait is bounded (2 s); one that gives up sets
 *   KD_DEV_TIMEOUT and records where in the control block.
 */
int kd_tree_verify_attn(const kd_bf16_t* q_nope_absorbed, const kd_bf16_t* q_rope,
                        const kd_bf16_t* c_kv, const kd_bf16_t* k_rope,
                        int64_t kv_row_stride_c, int64_t kv_row_stride_r, int64_t cap,
                        const int32_t* cache_lens, const uint32_t* vis,
                        const int32_t* positions, int B, int n, int H, float scale,
                        kd_bf16_t* out, float* lse, void* workspace, size_t ws_bytes,
                        int kv_splits, cudaStream_t stream);

/*
 * kd_tree_verify_attn_simt -- the same operation as kd_tree_verify_attn computed on
 * CUDA cores (one warp per node and head, keys streamed one at a time).  No
 * workspace, no tensor cores, far slower: it is a second, independent GPU
 * implementation that the tests use to cross-check the tensor-core kernel, not a
 * path to serve with.  Same arguments and checks; device errors go to `dev_error`
 * (may be NULL, in which case they are discarded).
 */
int kd_tree_verify_attn_simt(const kd_bf16_t* q_nope_absorbed, const kd_bf16_t* q_rope,
                             const kd_bf16_t* c_kv, const kd_bf16_t* k_rope,
                             int64_t kv_row_stride_c, int64_t kv_row_stride_r, int64_t cap,
                             const int32_t* cache_lens, const uint32_t* vis,
                             const int32_t* positions, int B, int n, int H, float scale,
                             kd_bf16_t* out, float* lse, int32_t* dev_error,
                             cudaStream_t stream);

/*
 * kd_tree_verify_attn_noalloc -- kd_tree_verify_attn for callers that cannot
 * allocate device memory at call time: code running under CUDA graph capture,
 * serving loops that keep allocator calls off the hot path, and C hosts without a
 * device allocator.  (The pages have no counterpart; this is an interface
 * convenience of this library.)
 *
 * Same inputs, outputs and checks as kd_tree_verify_attn, without the workspace
 * arguments.  The workspace is a fixed array of KD_NOALLOC_SCRATCH_BYTES inside the
 * library; every GPU that loads the library holds it until the process exits.
 *   - With kv_splits = 0 the split count is chosen so that the partials fit the
 *     array; an explicit kv_splits whose workspace would exceed it returns KD_ERANGE
 *     and enqueues nothing.
 *   - The call allocates nothing: no cudaMalloc/cudaFree and no allocating library
 *     routine.  After every argument check passed it enqueues a memset of the
 *     array's control block (and of its split tickets, when it splits), the
 *     attention kernel and, when dev_error is not NULL, a 4-byte device-to-device
 *     copy of this call's KD_DEV_* bits into *dev_error (overwritten, not ORed).
 *     With dev_error NULL this call's device errors are discarded.
 *   - All of it is capturable into a CUDA graph (after the first call, below); a
 *     replay re-runs the memsets, so a graph replays correctly any number of times.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and sets kernel attributes; make that first call before
 *     any stream capture.
 *   - All calls share the one array and it keeps the previous call's contents: calls
 *     whose kernels overlap on the GPU (e.g. on two streams without ordering between
 *     them) race on it and must be serialised by the caller.
 */
#define KD_NOALLOC_SCRATCH_BYTES (32 << 20)
int kd_tree_verify_attn_noalloc(const kd_bf16_t* q_nope_absorbed, const kd_bf16_t* q_rope,
                                const kd_bf16_t* c_kv, const kd_bf16_t* k_rope,
                                int64_t kv_row_stride_c, int64_t kv_row_stride_r, int64_t cap,
                                const int32_t* cache_lens, const uint32_t* vis,
                                const int32_t* positions, int B, int n, int H, float scale,
                                kd_bf16_t* out, float* lse, int kv_splits, int32_t* dev_error,
                                cudaStream_t stream);

/*
 * kd_tree_build -- best-first draft trees from per-depth drafter candidates, one per
 * request ("The Architecture of Pragmatic Ambition", section "The Knowledge
 * Architecture": the tree builder takes per-depth top-k candidates and constructs a
 * best-first tree).  The pages give no scoring rule; this is the reading taken:
 *   logp        [B][D][K] fp32: log-probabilities of depth d's K candidates, sorted
 *               from the most to the least likely (not checked; unsorted input gives
 *               the same deterministic steps, not a best-first tree); no NaN.
 *   cand_tokens [B][D][K] int32: the candidates' tokens.
 *   root_tokens [B] int32: the last verified token (node 0).
 *   A node's score is the float32 sum of log-probabilities along its path.  The
 *   tree is node 0 plus the n - 1 best nodes, popped best first from the frontier
 *   of the tree so far (ties: lower depth, then lower parent, then lower
 *   candidate); node index = pop order, so parents[i] < i.
 *   parents, tokens [B][n] int32 out (parents[b][0] = -1); depth [B][n] int32 and
 *   score [B][n] fp32 out, each optional (NULL).
 * Limits: 1 <= n <= 128, 1 <= D <= 4096, 1 <= K <= 255, and the candidates must
 * hold at least n - 1 nodes (K + K^2 + ... + K^D >= n - 1); otherwise KD_EINVAL.
 */
int kd_tree_build(const float* logp, const int32_t* cand_tokens, const int32_t* root_tokens,
                  int B, int D, int K, int n, int32_t* parents, int32_t* tokens, int32_t* depth,
                  float* score, cudaStream_t stream);

/*
 * kd_tree_accept -- greedy acceptance of B verified trees.
 *   node_tokens [B][n], parents [B][n], target_argmax [B][n] int32 (target_argmax[b][i]
 *   is the target's prediction after node i).
 *   Starting at the root, repeatedly step to the lowest-index child c of the current
 *   node with node_tokens[c] == target_argmax[current]; stop when none matches.
 *   path  [B][n] int32 out: path[b][0..len-1] = accepted nodes (path[b][0] = 0);
 *                 entries from len on are set to -1.
 *   len   [B]    int32 out: accepted count including the root (1 .. n).
 *   bonus [B]    int32 out: target_argmax[b][last accepted node].
 *   A bad parent array gives KD_DEV_BAD_PARENT and len = 1, path = {0}.
 */
int kd_tree_accept(const int32_t* node_tokens, const int32_t* parents,
                   const int32_t* target_argmax, int B, int n, int32_t* path,
                   int32_t* len, int32_t* bonus, int32_t* dev_error, cudaStream_t stream);

/*
 * kd_accept_workspace_bytes -- scratch bytes kd_tree_accept_logits needs for B
 * requests of n nodes (0 for invalid shapes).
 */
size_t kd_accept_workspace_bytes(int B, int n);

/*
 * kd_tree_accept_logits -- the target's greedy token after every node, taken from
 * its logits, fused with kd_tree_accept in one launch ("The Architecture of
 * Pragmatic Ambition", section "The Output Knowledge: What This Message Creates":
 * argmax is an engine primitive, and the speculative output must equal greedy
 * decoding token for token).
 *   logits [B][n][V] fp32, row pitch V, 16-byte aligned, V a multiple of 4 and
 *          at most 2^31 - 1 (V = 163840 for Kimi-K2).  Row (b, i) holds the
 *          target's logits after node i.
 *   target_argmax [B][n] int32 out, or NULL: index of the largest logit of each
 *          row; the lowest index among equal maxima, a NaN above every number
 *          (the first NaN wins), -0.0 equal to +0.0.
 *   node_tokens, parents, path, len, bonus: as kd_tree_accept, with these tokens.
 *   workspace: caller-owned device scratch of at least
 *          kd_accept_workspace_bytes(B, n) bytes, 16-byte aligned, cleared by the
 *          call; do not share it between calls that may overlap.
 * Returns KD_EINVAL for null or misaligned pointers, bad shapes or V; KD_ERANGE
 * if ws_bytes is too small.  A bad parent array sets KD_DEV_BAD_PARENT as
 * kd_tree_accept does.  The logits are read once (streaming loads).
 */
int kd_tree_accept_logits(const int32_t* node_tokens, const int32_t* parents,
                          const float* logits, int B, int n, int64_t V,
                          int32_t* target_argmax, int32_t* path, int32_t* len,
                          int32_t* bonus, void* workspace, size_t ws_bytes,
                          int32_t* dev_error, cudaStream_t stream);

/*
 * kd_kv_compact -- gather each request's accepted latents into contiguous slots.
 *   For j < len[b]: row L+j <- row L+path[b][j] of c_kv and k_rope (L = cache_lens[b]),
 *   all rows read before any is written; then cache_lens[b] += len[b].  Rows below L
 *   and from L+len on are untouched.  In place on c_kv, k_rope and cache_lens.
 *   A request with len not in [1, n], a path entry not in [0, n) or L + n > cap is
 *   left unchanged and sets KD_DEV_BAD_PATH / KD_DEV_CACHE_FULL.
 */
int kd_kv_compact(kd_bf16_t* c_kv, kd_bf16_t* k_rope, int64_t kv_row_stride_c,
                  int64_t kv_row_stride_r, int64_t cap, const int32_t* path,
                  const int32_t* len, int32_t* cache_lens, int B, int n,
                  int32_t* dev_error, cudaStream_t stream);

/*
 * kd_kv_write_nodes -- store the n node latents of each request at slots L..L+n-1.
 *   node_ckv [B][n][512], node_krope [B][n][64] bf16 contiguous.  cache_lens is not
 *   changed.  A request with L + n > cap is skipped and sets KD_DEV_CACHE_FULL.
 */
int kd_kv_write_nodes(kd_bf16_t* c_kv, kd_bf16_t* k_rope, int64_t kv_row_stride_c,
                      int64_t kv_row_stride_r, int64_t cap, const int32_t* cache_lens,
                      const kd_bf16_t* node_ckv, const kd_bf16_t* node_krope, int B,
                      int n, int32_t* dev_error, cudaStream_t stream);

/*
 * Paged caches.  A shared pool of pages of page_size slots replaces the per-request
 * contiguous cache (page size 1 fragments a live service's memory: "The
 * Architectural Keystone ...", "Assumptions Embedded in the Design").  Request b's
 * logical slot s is row page_table[b][s / page_size] * page_size + s % page_size of
 *   c_pages [num_pages * page_size][kv_row_stride_c] and
 *   r_pages [num_pages * page_size][kv_row_stride_r] (bf16),
 * page_table [B][pages_per_req] int32 (device), so a request holds
 * cap = pages_per_req * page_size logical slots.  Pages of different requests must
 * not overlap.  The calls below are the contiguous ones on that logical view; their
 * results are identical to running the contiguous calls on the gathered caches.
 */

/*
 * kd_tree_verify_attn_paged -- kd_tree_verify_attn over a paged cache.  page_size is
 * 64, 128 or 256 and pages_per_req at most 2047; the workspace is sized by
 * kd_verify_workspace_bytes(B, n, H, pages_per_req * page_size, kv_splits);
 * KD_EINVAL otherwise as the contiguous call.  A request whose pages
 * [0, ceil((L + n) / page_size)) hold an id outside [0, num_pages) sets
 * KD_DEV_BAD_PAGE and its out/lse rows are left untouched (the other requests are
 * computed normally).  A bad id never faults: the loads use page 0 in its place.
 */
int kd_tree_verify_attn_paged(const kd_bf16_t* q_nope_absorbed, const kd_bf16_t* q_rope,
                              const kd_bf16_t* c_pages, const kd_bf16_t* r_pages,
                              int64_t kv_row_stride_c, int64_t kv_row_stride_r, int page_size,
                              const int32_t* page_table, int64_t pages_per_req, int64_t num_pages,
                              const int32_t* cache_lens, const uint32_t* vis,
                              const int32_t* positions, int B, int n, int H, float scale,
                              kd_bf16_t* out, float* lse, void* workspace, size_t ws_bytes,
                              int kv_splits, cudaStream_t stream);

/*
 * kd_kv_write_nodes_paged / kd_kv_compact_paged -- kd_kv_write_nodes and
 * kd_kv_compact through a page table (any page_size >= 1).  A request whose slots
 * L..L+n-1 touch a page id outside [0, num_pages) is skipped and sets
 * KD_DEV_BAD_PAGE.  The compaction gathers rows inside the request's pages (the
 * page table itself is not rewritten).
 */
int kd_kv_write_nodes_paged(kd_bf16_t* c_pages, kd_bf16_t* r_pages, int64_t kv_row_stride_c,
                            int64_t kv_row_stride_r, int page_size, const int32_t* page_table,
                            int64_t pages_per_req, int64_t num_pages, const int32_t* cache_lens,
                            const kd_bf16_t* node_ckv, const kd_bf16_t* node_krope, int B, int n,
                            int32_t* dev_error, cudaStream_t stream);
int kd_kv_compact_paged(kd_bf16_t* c_pages, kd_bf16_t* r_pages, int64_t kv_row_stride_c,
                        int64_t kv_row_stride_r, int page_size, const int32_t* page_table,
                        int64_t pages_per_req, int64_t num_pages, const int32_t* path,
                        const int32_t* len, int32_t* cache_lens, int B, int n, int32_t* dev_error,
                        cudaStream_t stream);

/*
 * kd_read_device_error -- synchronises `stream`, returns the device error word
 * (>= 0, KD_DEV_* bits) and zeroes it when `clear` is non-zero.  Negative return =
 * KD_E* code of the copy itself.
 */
int kd_read_device_error(int32_t* dev_error, int clear, cudaStream_t stream);

/* kd_strerror -- static text for a KD_E* code (KD_ELAUNCH: last CUDA error text). */
const char* kd_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* KD_VERIFY_H */
