/*
 * medusa.h -- C ABI of libmedusa: the per-step Medusa draft-and-verify chain
 * on one NVIDIA B200 (sm_100a).
 *
 * The step, as "Medusa heads versus separate draft model" describes it
 * (sections "What each one is" and "Acceptance", tree paragraph):
 *   1. K draft heads read the target's last hidden state in a single
 *      parallel pass; head k applies a residual block and then a vocabulary
 *      projection of its own, drafting the token k places ahead;
 *   2. the heads' best-scoring candidates, combined, make up a tree;
 *   3. the target checks every branch at once under a tree-shaped attention
 *      mask;
 *   4. decoding continues along the longest matching branch.
 * Calls: md_medusa_heads (1), md_tree_build (2), md_tree_attention (3, one
 * attention layer of the verification pass), md_tree_accept (4).
 * md_hydra_draft does 1 and 2 with sequentially dependent (Hydra) heads.
 *
 * Conventions (all calls):
 *  - Tensor pointers are DEVICE pointers unless a comment says "host". The
 *    caller allocates and owns every buffer, including the workspace each
 *    call asks for; the library keeps no pointer after a call returns.
 *  - bf16 tensors are passed as uint16_t bit patterns (md_bf16).
 *  - Layouts are dense row-major in the index order written in brackets.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream). Outputs are ready when the stream reaches the
 *    call's point.
 *  - Shapes and pointers are checked on the host first; on error the call
 *    returns a negative md_status and launches nothing.
 *  - Errors that depend on device data (a prefix that does not fit the KV
 *    cache, a row or token id out of range) never trap: the kernels skip the
 *    offending item, write a defined value (-1 ids, zeros) and set a bit in a
 *    device status word read by md_get_device_status().
 *  - No C++ exception crosses this interface.
 *  - Kernels use no floating-point atomics: results are bitwise
 *    reproducible run to run for the same inputs and sizes.
 */
#ifndef MEDUSA_H
#define MEDUSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MD_API __attribute__((visibility("default")))
#else
#define MD_API
#endif

typedef int32_t md_status;
typedef uint16_t md_bf16;

enum {
  MD_OK = 0,
  MD_ERR_INVALID_ARG = -1, /* null pointer, non-positive size, bad tree spec     */
  MD_ERR_UNSUPPORTED = -2, /* valid but outside the supported ranges below      */
  MD_ERR_CUDA = -3,        /* a CUDA runtime call failed (launch, copy, ...)    */
  MD_ERR_WORKSPACE = -4,   /* workspace pointer null or smaller than required   */
  MD_ERR_TIMEOUT = -5      /* a bounded device wait gave up (device status bit) */
};

/* Bits of the device status word (md_get_device_status). */
enum {
  MD_DEV_BAD_PREFIX = 1,   /* prefix_len[b] < 0 or prefix_len[b] + T > S_max     */
  MD_DEV_BAD_ROW = 2,      /* head_row[b] outside [0, M)                         */
  MD_DEV_BAD_TOKEN = 4,    /* a token id outside [0, V) reached tree_accept or   */
                           /* a Hydra head input                                */
  MD_DEV_TIMEOUT = 8,      /* a pipeline wait exceeded its bound                 */
  MD_DEV_BAD_PATH = 16     /* md_tree_commit got a length or path that is not a  */
                           /* root-to-node path of the tree                       */
};

/* Supported ranges (anything else: MD_ERR_UNSUPPORTED).
 *   heads:     1 <= K <= 8, 1 <= k_i <= kmax <= 16, d % 64 == 0, V % 8 == 0,
 *              V >= 256, 1 <= M <= 4096 (M = 1: CUDA-core weight stream;
 *              2 <= M <= 32: tcgen05 weight stream with the weights as the
 *              MMA's M; M > 32: tcgen05 GEMM on 128-row tiles; from two rows
 *              h and b1 must be 16-byte aligned).
 *   tree:      1 <= T <= 128, depth <= K.
 *   attention: dh in {64, 128}, Hq % Hkv == 0, Hq / Hkv <= 16.
 */
#define MD_MAX_T 128
#define MD_MAX_K 8
#define MD_MAX_KMAX 16

/* ------------------------------------------------------------------------ */
/* Tree spec.                                                                */
/* ------------------------------------------------------------------------ */

/* Opaque, host-only description of a fixed candidate tree. */
typedef struct md_tree md_tree;

/* Creates a tree spec.
 * Source: "Medusa heads versus separate draft model", section "Acceptance",
 * tree paragraph (each head offers its best-scoring candidates and their
 * combinations make up the tree).
 *
 * Node 0 is the root (the token the target already emitted). A node at
 * depth k >= 1 is a candidate from head k: it holds head_rank[j], the rank
 * of its token in head k's top-k list.
 *
 * parent     host [T]: parent[0] = -1; 0 <= parent[j] < j for j >= 1.
 * head_rank  host [T]: head_rank[0] ignored; 0 <= head_rank[j] < k_per_head[depth(j)-1].
 * T          nodes including the root, 1..MD_MAX_T.
 * K          number of heads; every depth must be <= K.
 * k_per_head host [K]: top-k of each head.
 * out        receives a handle; free it with md_tree_destroy.
 * Two children of one node must not share a rank (their tokens would be
 * equal). The spec is copied; the arrays may be freed after the call.
 * Allocates host memory only. Errors: MD_ERR_INVALID_ARG for any violation. */
MD_API md_status md_tree_create(const int32_t* parent, const int32_t* head_rank, int32_t T, int32_t K,
                         const int32_t* k_per_head, md_tree** out);
MD_API md_status md_tree_destroy(md_tree* tree);
/* T and the deepest depth of a tree (either pointer may be NULL). */
MD_API md_status md_tree_info(const md_tree* tree, int32_t* T, int32_t* max_depth);

/* ------------------------------------------------------------------------ */
/* 1. Draft heads with fused per-head top-k.                                 */
/* ------------------------------------------------------------------------ */

/* Workspace bytes md_medusa_heads needs for these sizes. */
MD_API md_status md_heads_workspace(int32_t M, int32_t d, int32_t V, int32_t K, int32_t kmax, size_t* bytes);

/* The K Medusa heads on M hidden rows, fused with a top-k per head.
 * Source: "Medusa heads versus separate draft model", sections "What each
 * one is" (per head a residual block, then a vocabulary projection of its
 * own; all heads read the same hidden state in one parallel pass) and "Cost
 * per step" (a d x d layer with bias in the block; a bias-free d x V
 * projection).
 *
 *   u[m,k,o]      = b1[k,o] + sum_i h[m,i] * W1[k,i,o]          (fp32 accumulate)
 *   z[m,k,o]      = bf16_rne( h[m,o] + u / (1 + exp(-u)) )        (SiLU residual)
 *   logit[m,k,v]  = sum_i z[m,k,i] * Wv[k,i,v]                   (fp32 accumulate)
 *   topk_*[m,k,:] = the k_per_head[k] largest logits of row (m,k), ordered
 *                   by (value descending, id ascending); slots past
 *                   k_per_head[k] hold id -1 and value -inf.
 *
 * h          [M, d] bf16.        W1 [K, d, d] bf16 (input-major: W1[k][i][o]).
 * b1         [K, d] bf16.        Wv [K, d, V] bf16 (input-major: Wv[k][i][v]).
 * k_per_head host [K].           kmax: stride of the top-k outputs (>= every k_i).
 * topk_ids   [M, K, kmax] int32, topk_vals [M, K, kmax] fp32 (outputs).
 * logits_dbg [M, K, V] fp32 or NULL: when given, the full logits are also
 *            written (debug / parity only; the fused path never needs them).
 * ws, ws_bytes: workspace of at least md_heads_workspace() bytes, any
 *   contents: nothing in it needs clearing before a call (the kernels'
 *   arrival tickets carry a per-call epoch), and one workspace serves call
 *   after call on one stream.
 * Errors: MD_ERR_INVALID_ARG, MD_ERR_UNSUPPORTED, MD_ERR_WORKSPACE, MD_ERR_CUDA. */
MD_API md_status md_medusa_heads(const md_bf16* h, const md_bf16* W1, const md_bf16* b1, const md_bf16* Wv,
                          int32_t M, int32_t d, int32_t V, int32_t K, const int32_t* k_per_head,
                          int32_t kmax, int32_t* topk_ids, float* topk_vals, float* logits_dbg,
                          void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes md_medusa_heads_shared needs for these sizes. */
MD_API md_status md_heads_shared_workspace(int32_t M, int32_t d, int32_t V, int32_t K, int32_t kmax, size_t* bytes);

/* The K heads with ONE vocabulary projection shared by all of them.
 * Source: "Medusa heads versus separate draft model", section "What
 * interviewers probe next": each head normally has its own d x V projection
 * (initialised from the LM head); sharing one saves (K - 1) d V parameters
 * (3.15B of them for four heads at d = 8,192, V = 128,256) and costs some
 * acceptance. The residual blocks stay per head:
 *   z[m,k,:]     = bf16_rne( h[m,:] + SiLU(h[m,:] W1[k] + b1[k]) )
 *   logit[m,k,v] = sum_i z[m,k,i] * Wv[i,v]
 * and the top-k is as in md_medusa_heads. Arguments as md_medusa_heads except
 * Wv [d, V] bf16 (16-byte aligned, as are h and b1). The projection is
 * streamed once for all heads: 2 d V bytes instead of 2 K d V.
 * Errors: as md_medusa_heads. */
MD_API md_status md_medusa_heads_shared(const md_bf16* h, const md_bf16* W1, const md_bf16* b1,
                                        const md_bf16* Wv, int32_t M, int32_t d, int32_t V, int32_t K,
                                        const int32_t* k_per_head, int32_t kmax, int32_t* topk_ids,
                                        float* topk_vals, float* logits_dbg, void* ws, size_t ws_bytes,
                                        void* stream);

/* The draft heads with SAMPLED candidates: each head's k candidates are k
 * draws without replacement from its own distribution
 * q = softmax(logits / temperature), in draw order, instead of its top-k.
 * Source: "Medusa heads versus separate draft model", section "Training"
 * (rejection sampling keeps the target's distribution exactly; it needs drafts
 * drawn from a known distribution, which md_tree_accept_rejection then uses).
 *
 * The draws use the Gumbel-top-k construction: with one caller-supplied
 * uniform u in (0, 1) per (row, head, token),
 *   key[m,k,v] = logit[m,k,v] / temperature - ln(-ln u[m,k,v]),
 * and the candidates are the k_per_head[k] tokens of largest key, by key
 * descending (ties to the lower id). The i-th candidate is then distributed as
 * q restricted to the tokens not drawn before it. u = 0 or 1 gives a key of
 * -inf or +inf.
 *
 *   uniforms   [M, K, V] fp32 (16-byte aligned), read once
 *   topk_ids   [M, K, kmax] int32, the candidates in draw order (-1 padded)
 *   topk_keys  [M, K, kmax] fp32, their keys (-inf padded)
 *   logits     [M, K, V] fp32 (required, 16-byte aligned): the heads' logits,
 *              which md_tree_accept_rejection reads as the draft distribution
 * Everything else, the workspace (md_heads_workspace) and the errors are as
 * md_medusa_heads; temperature must be positive and finite. */
MD_API md_status md_medusa_heads_sampled(const md_bf16* h, const md_bf16* W1, const md_bf16* b1,
                                         const md_bf16* Wv, int32_t M, int32_t d, int32_t V, int32_t K,
                                         const int32_t* k_per_head, int32_t kmax, float temperature,
                                         const float* uniforms, int32_t* topk_ids, float* topk_keys, float* logits,
                                         void* ws, size_t ws_bytes, void* stream);

/* Size of the library-owned scratch behind md_medusa_heads_static (32 MiB). */
#define MD_HEADS_STATIC_SCRATCH_BYTES (32u << 20)

/* md_medusa_heads for callers that cannot allocate device memory.
 * (An addition of this library: the pages have no counterpart.)
 *
 * Some callers have no way to hand the library a workspace: runtimes whose
 * device memory is owned by a pool that no plugin may grow, or latency-bound
 * decode loops that must never reach the allocator (cudaMalloc and cudaFree
 * can synchronise the device and can fail for lack of memory at an
 * unpredictable point). This entry point computes exactly what
 * md_medusa_heads computes, with the same arguments minus the workspace: its
 * scratch is a fixed MD_HEADS_STATIC_SCRATCH_BYTES array inside the
 * library's device image, which every GPU that loads the library keeps until
 * the process exits. It calls no cudaMalloc, cudaFree or other allocating
 * routine. The caller still provides the inputs and outputs.
 *
 * - Arguments are checked as md_medusa_heads checks them first; then sizes
 *   whose scratch (md_heads_workspace on the calling device) exceeds the
 *   array are rejected with MD_ERR_WORKSPACE before anything is launched. The
 *   scratch of the tensor-core path grows with the device's SM count, so the
 *   largest admitted M depends on the GPU: on a 148-SM B200 at d = 8192,
 *   V = 128256, K = 4, kmax = 10 every M up to 433 fits. Callers that need a guarantee
 *   compare md_heads_workspace(...) with MD_HEADS_STATIC_SCRATCH_BYTES on
 *   their device.
 * - The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture on the device.
 * - Every call on a device shares the one array and leaves its contents
 *   behind and needs nothing cleared (the heads kernels' tickets carry a
 *   per-call epoch). Two calls whose
 *   kernels overlap on the GPU (different streams, no ordering between them)
 *   race on the array and give undefined results: order them on one stream
 *   or with events.
 * Errors: as md_medusa_heads, plus MD_ERR_WORKSPACE for oversized shapes. */
MD_API md_status md_medusa_heads_static(const md_bf16* h, const md_bf16* W1, const md_bf16* b1,
                                        const md_bf16* Wv, int32_t M, int32_t d, int32_t V, int32_t K,
                                        const int32_t* k_per_head, int32_t kmax, int32_t* topk_ids,
                                        float* topk_vals, float* logits_dbg, void* stream);

/* ------------------------------------------------------------------------ */
/* 2. Candidate tree construction.                                           */
/* ------------------------------------------------------------------------ */

/* Tokens, parents, ancestor mask and position ids of the tree for B requests.
 * Source: "Medusa heads versus separate draft model", section "Acceptance",
 * tree paragraph.
 *
 *   tokens[b,0] = root_token[b];
 *   tokens[b,j] = topk_ids[row_b, depth(j)-1, head_rank[j]]  (j >= 1),
 *                 row_b = head_row ? head_row[b] : b;
 *   parent[j]   = the tree's parent array (root -1);
 *   anc[j,w]    bit (i % 32) of word w = i / 32 is set iff node i is an
 *               ancestor of j or j itself (W = ceil(T/32) words per node);
 *   pos[b,j]    = prefix_len[b] + depth(j)   (position id for the target's
 *               rotary embedding; the KV slot of node j is prefix_len[b] + j).
 *
 * topk_ids [M, K, kmax] int32 from md_medusa_heads.  head_row [B] int32 or NULL.
 * root_token [B] int32.  prefix_len [B] int32.
 * tokens [B, T] int32, parent [T] int32, anc [T, W] uint32, pos [B, T] int32.
 * A head_row outside [0, M) sets MD_DEV_BAD_ROW and that request's candidate
 * tokens are -1. Errors: MD_ERR_INVALID_ARG, MD_ERR_CUDA. */
MD_API md_status md_tree_build(const md_tree* tree, const int32_t* topk_ids, int32_t M, int32_t kmax,
                        const int32_t* head_row, const int32_t* root_token, const int32_t* prefix_len,
                        int32_t B, int32_t* tokens, int32_t* parent, uint32_t* anc, int32_t* pos,
                        void* stream);

/* ------------------------------------------------------------------------ */
/* 1+2 (sequentially dependent heads). Hydra drafting of the whole tree.     */
/* ------------------------------------------------------------------------ */

/* Workspace bytes md_hydra_draft needs for this tree and these sizes. */
MD_API md_status md_hydra_workspace(const md_tree* tree, int32_t B, int32_t d, int32_t V, int32_t kmax,
                                    size_t* bytes);

/* Drafts every node of the tree with sequentially dependent heads, then
 * writes the tree outputs of md_tree_build.
 * Sources: "Medusa heads versus separate draft model", section "Acceptance"
 * (a Medusa head drafts without knowing the earlier heads' guesses);
 * "Hydra: Sequentially-Dependent Draft Heads for Medusa Decoding" (abstract:
 * drop-in draft heads whose guesses are conditioned on the earlier tokens of
 * the candidate continuation). The pages give no Hydra architecture; this
 * call reads it as the Medusa head of md_medusa_heads applied to the hidden
 * state plus the input embedding of the parent node's token:
 *
 *   x_p           = bf16_rne( h[row_b] + E[tokens[b,p]] )   (exact sum, one rounding)
 *   head l        = the residual block and projection of md_medusa_heads with
 *                   W1[l], b1[l], Wv[l], applied to x_p for every node p at
 *                   depth l that has children, top-k_l fused;
 *   tokens[b,j]   = entry head_rank[j] of that top-k of x_parent(j);
 *   tokens[b,0]   = root_token[b]; parent, anc, pos as md_tree_build.
 *
 * The heads run depth by depth (depth l needs the tokens of depth l), each
 * level on B * n_l rows (n_l = nodes at depth l with children).
 *
 * tree       the spec; K must equal the K it was created with.
 * h          [M, d] bf16; row_b = head_row ? head_row[b] : b (head_row [B] or NULL).
 * E          [V, d] bf16 input token embedding of the target.
 * W1 [K, d, d], b1 [K, d], Wv [K, d, V] bf16 as md_medusa_heads; h, E, W1,
 *            b1 and Wv 16-byte aligned.
 * kmax       >= every k of the tree's k_per_head.
 * root_token [B], prefix_len [B] int32.
 * tokens [B, T], parent [T], anc [T, W] uint32, pos [B, T] (outputs).
 * logits_dbg NULL, or fp32 [rows, V] with rows = B * (n_0 + ... + n_{L-1}):
 *            when given, the logits of every head row are also written
 *            (debug / parity only), level by level, within a level request
 *            by request, within a request the depth-l nodes with children
 *            in node order.
 * ws, ws_bytes: workspace of at least md_hydra_workspace() bytes, 256-byte aligned.
 * A head_row outside [0, M) sets MD_DEV_BAD_ROW (that request's head inputs
 * use a zero hidden state); a drafted token outside [0, V) sets
 * MD_DEV_BAD_TOKEN (its embedding counts as zero).
 * Errors: MD_ERR_INVALID_ARG, MD_ERR_UNSUPPORTED (sizes md_medusa_heads does
 * not take for one head on B * n_l rows), MD_ERR_WORKSPACE, MD_ERR_CUDA. */
MD_API md_status md_hydra_draft(const md_tree* tree, const md_bf16* h, int32_t M, const int32_t* head_row,
                                const md_bf16* E, const md_bf16* W1, const md_bf16* b1, const md_bf16* Wv,
                                int32_t d, int32_t V, int32_t K, int32_t kmax, const int32_t* root_token,
                                const int32_t* prefix_len, int32_t B, int32_t* tokens, int32_t* parent,
                                uint32_t* anc, int32_t* pos, float* logits_dbg, void* ws, size_t ws_bytes,
                                void* stream);

/* ------------------------------------------------------------------------ */
/* 3. Tree-masked attention (one layer of the verification pass).            */
/* ------------------------------------------------------------------------ */

MD_API md_status md_attention_workspace(int32_t B, int32_t T, int32_t Hq, int32_t Hkv, int32_t dh,
                                 int32_t S_max, size_t* bytes);

/* Attention of the T tree tokens over the KV prefix plus the tree.
 * Source: "Medusa heads versus separate draft model", section "Acceptance",
 * tree paragraph (every branch is checked in a single target pass under a
 * tree-shaped attention mask).
 *
 *   out[b,t,h,:] = sum_j softmax_j( scale * q[b,t,h,:] . K[b,g,j,:] ) V[b,g,j,:]
 *   over key slots j in [0, P_b) and P_b + a for every ancestor a of t
 *   (t included), with P_b = prefix_len[b] and KV head g = h / (Hq / Hkv).
 *
 * q       [B, T, Hq, dh] bf16 (already rotated by the caller).
 * k_cache, v_cache [B, Hkv, S_max, dh] bf16; slots [P_b, P_b + T) hold the
 *         tree tokens' own K/V (node j at slot P_b + j).
 * prefix_len [B] int32; P_b + T > S_max or P_b < 0 sets MD_DEV_BAD_PREFIX
 *         and writes zeros for that request.
 * scale   softmax scale; 0 means 1/sqrt(dh).
 * out     [B, T, Hq, dh] fp32.
 * Errors: MD_ERR_INVALID_ARG, MD_ERR_UNSUPPORTED, MD_ERR_WORKSPACE, MD_ERR_CUDA. */
MD_API md_status md_tree_attention(const md_bf16* q, const md_bf16* k_cache, const md_bf16* v_cache,
                            const int32_t* prefix_len, int32_t S_max, const md_tree* tree, int32_t B,
                            int32_t Hq, int32_t Hkv, int32_t dh, float scale, float* out, void* ws,
                            size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* 4. Acceptance of the longest matching branch.                             */
/* ------------------------------------------------------------------------ */

enum { MD_ACCEPT_GREEDY = 0, MD_ACCEPT_TYPICAL = 1 };

MD_API md_status md_accept_workspace(int32_t B, int32_t T, int32_t V, size_t* bytes);

/* Longest accepted root-to-node path per request, and the bonus token.
 * Source: "Medusa heads versus separate draft model", section "Acceptance",
 * tree paragraph (decoding continues along the branch that matches), and
 * section "Training" (typical acceptance: accepts more drafts, not lossless).
 *
 * Row t of logits is the target's distribution for the token after node t.
 * Non-root node j passes when
 *   greedy : tokens[b,j] == argmax_v logits[b,parent(j),v]  (lowest id on ties)
 *   typical: p(tokens[b,j]) > min(eps, alpha * exp(-H)), where p = softmax of
 *            logits[b,parent(j),:] / temperature and H is its entropy (nats).
 * A node is accepted when it and all its ancestors below the root pass.
 * accept_len[b] = L, the deepest accepted depth (0..max depth);
 * path[b, 0..L] = root .. the accepted depth-L node with the smallest index,
 *                 path[b, L+1..K] = -1 (K = the heads, the tree's max depth);
 * bonus[b]      = argmax of the last accepted node's row (lowest id on ties).
 *
 * logits [B, T, V] fp32.  tokens [B, T] int32 (from md_tree_build).
 * K      width of `path` minus one (>= the tree's max depth).
 * accept_len [B], path [B, K+1], bonus [B] int32 (outputs).
 * Errors: MD_ERR_INVALID_ARG, MD_ERR_UNSUPPORTED, MD_ERR_WORKSPACE, MD_ERR_CUDA. */
MD_API md_status md_tree_accept(const float* logits, int32_t V, const int32_t* tokens, const md_tree* tree,
                         int32_t B, int32_t K, int32_t mode, float temperature, float eps, float alpha,
                         int32_t* accept_len, int32_t* path, int32_t* bonus, void* ws, size_t ws_bytes,
                         void* stream);


/* Sampled (lossless) acceptance: the emitted tokens follow the target's own
 * sampling distribution.
 * Source: "Medusa heads versus separate draft model", section "Training" (when
 * the target distribution must be kept exactly, the page recommends rejection
 * sampling instead of typical acceptance); it gives no algorithm for a tree of
 * deterministic top-k candidates. Reading: rejection sampling of a candidate chosen with
 * certainty (a point-mass draft) accepts it with probability p(c) and else
 * samples p with c removed; over a node's candidate children this is one draw
 * y_t ~ p_t of the node's row, accepting the child whose token is y_t.
 *
 *   p_t = softmax(logits[b,t,:] / temperature)
 *   y_t = min{ v : sum_{w <= v} p_t(w) > uniforms[b,t] }   (ids in order)
 *   non-root node j passes iff tokens[b,j] == y_{parent(j)}; the path rule is
 *   md_tree_accept's; bonus[b] = y of the last accepted node.
 *
 * uniforms [B, T] fp32 in [0, 1), device: the random numbers are the caller's
 *          (one per tree row), so runs are reproducible.
 * temperature > 0. V <= 2,097,152 and V % 8 == 0. Other arguments as for
 * md_tree_accept; the workspace is md_accept_workspace's. Draws are made in
 * fp32 with fixed summation order: a uniform within ~1e-5 (relative) of a CDF
 * boundary may resolve to the neighbouring id compared with exact arithmetic.
 * A token outside [0, V) never matches a draw.
 * Errors: MD_ERR_INVALID_ARG, MD_ERR_UNSUPPORTED, MD_ERR_WORKSPACE, MD_ERR_CUDA. */
MD_API md_status md_tree_accept_sampled(const float* logits, int32_t V, const int32_t* tokens, const md_tree* tree,
                                        int32_t B, int32_t K, float temperature, const float* uniforms,
                                        int32_t* accept_len, int32_t* path, int32_t* bonus, void* ws,
                                        size_t ws_bytes, void* stream);

/* Lossless acceptance of SAMPLED drafts (md_medusa_heads_sampled): rejection
 * sampling against the heads' own distributions, so the emitted tokens follow
 * the target's sampling distribution exactly.
 * Source: "Medusa heads versus separate draft model", section "Training"
 * (rejection sampling when the target distribution must be kept). The page
 * gives no algorithm for a tree; reading (recursive rejection over the
 * children of a node, drafts drawn without replacement):
 *
 *   At node t (root first) with target p = softmax(logits[b,t,:] / temperature)
 *   and children c_1..c_m carrying head ranks 0..m-1 (tokens y_1..y_m, the
 *   first m draws of head depth(t)), with that head's
 *   q = softmax(head_logits[head_row[b], depth(t), :] / temperature_q):
 *     r_1 = p; for i = 1..m: q_i = q without y_1..y_{i-1}, renormalised;
 *       accept c_i iff u_accept[b,c_i] < r_i(y_i) / q_i(y_i);
 *       else r_{i+1} = max(0, r_i - q_i) / sum max(0, r_i - q_i).
 *   An accepted child's token is emitted and the walk continues there. If no
 *   child is accepted, or t has no children, bonus[b] is drawn from r_{m+1}
 *   (p at a leaf) by inverse CDF in id order with u_residual[b,t], and the
 *   walk stops. accept_len[b] = accepted nodes; path[b] = root then the
 *   accepted nodes, -1 padded to K + 1.
 *
 *   logits       [B, T, V] fp32 target logits, row t = after node t
 *   tokens       [B, T] int32, from md_tree_build on md_medusa_heads_sampled's ids
 *   head_logits  [M, Kh, V] fp32, md_medusa_heads_sampled's logits output
 *   head_row     [B] int32 or NULL (request b uses row b): the heads row whose
 *                draws built request b's tree
 *   u_accept, u_residual  [B, T] fp32 uniforms in [0, 1), the caller's
 *   temperature, temperature_q > 0: of the target and of the draft heads
 * Every node's children must carry the ranks 0..m-1 (MD_ERR_UNSUPPORTED
 * otherwise); K >= tree depth, Kh >= tree depth; V <= 196,608. One 8-CTA
 * cluster per request; no workspace. Decisions are taken in fp32 with a fixed
 * summation order: a uniform within ~1e-5 (relative) of its threshold or CDF
 * boundary may resolve differently from exact arithmetic. A head row outside
 * [0, M) (MD_DEV_BAD_ROW) accepts nothing; a token outside [0, V)
 * (MD_DEV_BAD_TOKEN) is rejected.
 * Errors: MD_ERR_INVALID_ARG, MD_ERR_UNSUPPORTED, MD_ERR_CUDA. */
MD_API md_status md_tree_accept_rejection(const float* logits, int32_t V, const int32_t* tokens,
                                          const md_tree* tree, int32_t B, int32_t K, float temperature,
                                          const float* head_logits, int32_t M, int32_t Kh, const int32_t* head_row,
                                          float temperature_q, const float* u_accept, const float* u_residual,
                                          int32_t* accept_len, int32_t* path, int32_t* bonus, void* stream);

/* ------------------------------------------------------------------------ */
/* 5. Advancing along the accepted branch.                                   */
/* ------------------------------------------------------------------------ */

/* KV compaction and the next step's inputs, after md_tree_accept.
 * Source: "Medusa heads versus separate draft model", section "Acceptance",
 * tree paragraph (decoding continues along the branch that matches).
 *
 * For request b with P = prefix_len[b], L = accept_len[b], path = path[b]:
 *   K/V slot P + i  <-  K/V slot P + path[i]      (i = 0..L, in place; other
 *                                                  slots are left unchanged)
 *   new_prefix_len[b] = P + L + 1    (the root and the L accepted tokens)
 *   next_root[b]      = bonus[b]
 *   next_head_row[b]  = b * T + path[L]   (row of the last accepted node when
 *                                          the heads ran on all B * T nodes)
 *
 * k_cache, v_cache [B, Hkv, S_max, dh] bf16 (updated in place).
 * prefix_len [B] is read only; new_prefix_len [B] must be a different buffer.
 * accept_len [B], path [B, K+1], bonus [B] from md_tree_accept (K = its K).
 * A length or path that is not a root-to-node path of the tree, or a prefix
 * that does not fit, sets MD_DEV_BAD_PATH and leaves that request's cache
 * unchanged (new_prefix_len = P, next_head_row = -1).
 * Errors: MD_ERR_INVALID_ARG, MD_ERR_UNSUPPORTED (dh not 64/128), MD_ERR_CUDA. */
MD_API md_status md_tree_commit(md_bf16* k_cache, md_bf16* v_cache, int32_t S_max, int32_t Hkv, int32_t dh,
                                const md_tree* tree, int32_t B, const int32_t* prefix_len,
                                const int32_t* accept_len, const int32_t* path, int32_t K, const int32_t* bonus,
                                int32_t* new_prefix_len, int32_t* next_root, int32_t* next_head_row,
                                void* stream);

/* ------------------------------------------------------------------------ */
/* Status.                                                                   */
/* ------------------------------------------------------------------------ */

/* Synchronises `stream`, then stores the device status word (MD_DEV_* bits
 * set by kernels since the last clear) in *out; clears it if `clear` != 0. */
MD_API md_status md_get_device_status(void* stream, int32_t* out, int32_t clear);

/* Bound, in nanoseconds, on every pipeline wait of the library's kernels on
 * the current device (0: the default, 2 s). A correct launch never comes near
 * it; a wait that runs out flags MD_DEV_TIMEOUT and its kernel winds down and
 * returns, leaving the context usable. Synchronous (a copy to device memory);
 * affects kernels launched afterwards.
 * Errors: MD_ERR_CUDA. */
MD_API md_status md_set_wait_limit(uint64_t ns);

/* Test hook for the timeout path (not for production use): while chunk >= 0,
 * the producers of md_tree_attention's tensor-core kernel do not issue the K/V
 * copies of that chunk (counted from 0 in each CTA's work range), so the waits
 * that need them run out after md_set_wait_limit's bound: the call flags
 * MD_DEV_TIMEOUT, every copy that was issued lands before its CTA exits, every
 * tensor-core operation completes before TMEM is released, and the next call
 * without the hook is correct. chunk = -1 turns it off. Synchronous.
 * Errors: MD_ERR_INVALID_ARG (chunk < -1), MD_ERR_CUDA. */
MD_API md_status md_test_withhold_attention_chunk(int32_t chunk);

/* Diagnostic: reads bytes of device memory once, front to back in 16-byte
 * non-allocating loads (8 in flight per thread, 4 CTAs of 512 threads per SM),
 * and folds them into *sink (device, 4 bytes; written only for one particular
 * XOR value, so that the loads are kept). It measures the read-only bandwidth
 * that bounds the weight-stream kernels of md_medusa_heads (a copy moves every
 * byte twice and is not their ceiling). buf 16-byte aligned; bytes a multiple
 * of 16. Asynchronous on stream.
 * Errors: MD_ERR_INVALID_ARG (null, misaligned or ragged size), MD_ERR_CUDA. */
MD_API md_status md_stream_read(const void* buf, size_t bytes, uint32_t* sink, void* stream);

/* Static description of a status code. */
MD_API const char* md_status_string(md_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
MD_API int32_t md_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MEDUSA_H */
