/*
 * longspec_hta.h -- C ABI of Hybrid Tree Attention on B200 (sm_100a).
 *
 * Hybrid Tree Attention is the verification attention of LongSpec's
 * long-context speculative decoding.  For every query head, T speculated
 * tree tokens attend
 *   - to the long shared prefix KV cache, with no mask, and
 *   - to each other, under the tree mask: a token sees itself and its
 *     ancestors (parent[] chain up to -1, which stands for the prefix end).
 * The prefix part and the tree part are computed as two softmax partials and
 * merged exactly by log-sum-exp rescaling.
 *
 * Passages that define the operation:
 *   - LongSpec README (sail-sg/LongSpec), "Introduction", contribution
 *     "Hybrid Attention Aggregation": fast prefix computation combined with
 *     standard attention for tree mask handling.
 *   - LongSpec paper summary (Elamur Research), "Summary", Hybrid Tree
 *     Attention bullet: verification split into a Flash Attention pass over
 *     the prefix and a kernel for the speculated tree; "Key points": target
 *     attention latency 49.92 ms -> 12.54 ms (hardware not given).
 *   - LongSpec arXiv abstract (original English abstract): attention
 *     aggregation combining fast prefix implementations with standard
 *     attention for tree mask handling; lossless (title).
 *   - SpecExtend abstract (codewithpapers.app): Hybrid Tree Attention used as
 *     a drop-in attention component.
 *
 * Conventions shared by every entry point
 *   Layouts (row-major, no padding, all little-endian):
 *     q          bf16  [B][Hq][T][D]
 *     k_prefix   bf16  [B][Hkv][L_cap][D]     key j of sequence b valid for j < L_b
 *     v_prefix   bf16  [B][Hkv][L_cap][D]
 *     prefix_len int32 [B]                    0 <= L_b <= L_cap
 *     k_tree     bf16  [B][Hkv][T][D]
 *     v_tree     bf16  [B][Hkv][T][D]
 *     parent     int32 [B][T]                 parent[i] in [-1, i); -1 = child of the prefix end
 *     out        bf16  [B][Hq][T][D]
 *     lse        fp32  [B][Hq][T]             natural log of sum exp(scale * q.k) over visible keys
 *   Query head h reads KV head h / (Hq / Hkv) (contiguous GQA groups).
 *   Device pointers unless stated; every pointer 16-byte aligned.
 *   Ownership: the caller owns every buffer, the workspace included; the
 *   library allocates no device memory in any call.
 *   Streams: calls are asynchronous on `stream` (0 = legacy default stream);
 *   only longspec_hta_get_status synchronises.
 *   Return value: LONGSPEC_HTA_OK (0) or a negative longspec_hta_status.  A
 *   call that returns an error launched nothing.  Problems only the device
 *   can see (bad parent[], prefix_len out of range, a pipeline wait that ran
 *   out) are recorded in the workspace status word, reported by
 *   longspec_hta_get_status; the affected rows of `out`/`lse` are NaN.
 *   Limits: D in {64, 128}; 1 <= T <= LONGSPEC_HTA_T_MAX; Hq % Hkv == 0;
 *   B*Hq*T rows and B*Hkv*L_cap keys below 2^31.  No CPU fallback: on a
 *   device other than sm_100 the calls return LONGSPEC_HTA_ERR_UNSUPPORTED_DEVICE.
 */
#ifndef LONGSPEC_HTA_H
#define LONGSPEC_HTA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LONGSPEC_HTA_API __attribute__((visibility("default")))
#else
#define LONGSPEC_HTA_API
#endif

#define LONGSPEC_HTA_T_MAX 256
#define LONGSPEC_HTA_ABI_VERSION 1

typedef enum {
    LONGSPEC_HTA_OK = 0,
    LONGSPEC_HTA_ERR_INVALID_DIMS = -1,        /* sizes out of range, Hq % Hkv != 0, bad scale */
    LONGSPEC_HTA_ERR_NULL_POINTER = -2,
    LONGSPEC_HTA_ERR_MISALIGNED = -3,          /* a pointer not 16-byte aligned */
    LONGSPEC_HTA_ERR_T_TOO_LARGE = -4,         /* T > LONGSPEC_HTA_T_MAX */
    LONGSPEC_HTA_ERR_UNSUPPORTED_D = -5,       /* D not 64 or 128 */
    LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL = -6,
    LONGSPEC_HTA_ERR_CUDA = -7,                /* a CUDA runtime/driver call failed */
    LONGSPEC_HTA_ERR_UNSUPPORTED_DEVICE = -8,  /* current device is not sm_100 */
    LONGSPEC_HTA_ERR_INVALID_OPTION = -9,
    /* device-detected, reported by longspec_hta_get_status */
    LONGSPEC_HTA_ERR_BAD_PARENT = -16,         /* some parent[b][i] outside [-1, i) */
    LONGSPEC_HTA_ERR_PREFIX_LEN_RANGE = -17,   /* some prefix_len[b] outside [0, L_cap] */
    LONGSPEC_HTA_ERR_PIPELINE_TIMEOUT = -18,   /* a bounded in-kernel wait ran out */
    LONGSPEC_HTA_ERR_INTERNAL = -19,           /* a kernel precondition failed (a library bug) */
    LONGSPEC_HTA_ERR_BAD_BLOCK = -20,          /* a block_table entry outside [0, num_blocks) */
    LONGSPEC_HTA_ERR_BAD_PATH = -21            /* accept_len outside [0, T] or a path entry outside [0, T) */
} longspec_hta_status;

/* Problem sizes of one call.  scale 0 means 1/sqrt(D); otherwise > 0. */
typedef struct {
    int B, Hq, Hkv, D, T, L_cap;
    float scale;
} longspec_hta_dims;

/* Prefix kernels selectable through longspec_hta_options.prefix_kernel. */
#define LONGSPEC_HTA_PREFIX_TCGEN05 0   /* TMA + tcgen05/TMEM split-KV kernel (default) */
#define LONGSPEC_HTA_PREFIX_SIMT    1   /* plain CUDA-core split-KV kernel, for cross-checks */

/* Optional knobs of longspec_hta_verify_ex.  Zero-initialise for defaults. */
typedef struct {
    int num_splits;          /* prefix split-KV chunks per (b, KV head), at most 64 (larger
                                requests are clamped); 0 = chosen by the library */
    int prefix_kernel;       /* LONGSPEC_HTA_PREFIX_* */
    cudaEvent_t prefix_begin;/* if non-null, recorded on `stream` right before the prefix kernel */
    cudaEvent_t prefix_end;  /* if non-null, recorded on `stream` right after the prefix kernel */
} longspec_hta_options;

/* A paged prefix KV cache (the block-table layout of serving engines): the
 * keys of sequence b are cut into blocks of block_size consecutive
 * positions; block_table[b][i] names the cache block that holds positions
 * [i*block_size, (i+1)*block_size) of sequence b for every KV head.
 *   k_cache, v_cache: bf16 [num_blocks][Hkv][block_size][D], device, 16-byte
 *                     aligned; block n, KV head h, position p at
 *                     ((n*Hkv + h)*block_size + p)*D.
 *   block_table:      int32 [B][max_blocks], device; entries past the last
 *                     block a sequence uses are not read.
 *   block_size:       16, 32, 64 or 128.
 *   max_blocks:       >= ceil(L_cap / block_size).
 * An entry outside [0, num_blocks) is read as block 0 and reported by
 * longspec_hta_get_status as LONGSPEC_HTA_ERR_BAD_BLOCK. */
typedef struct {
    const void *k_cache;
    const void *v_cache;
    const int32_t *block_table;
    int num_blocks;
    int block_size;
    int max_blocks;
} longspec_hta_paged_kv;

/* ABI version of the loaded library (LONGSPEC_HTA_ABI_VERSION). */
LONGSPEC_HTA_API int longspec_hta_abi_version(void);

/* Build-time tuning of the loaded library, as "key=value" pairs separated
 * by spaces: kv_stages_d128 (K/V ring depth of the tcgen05 prefix kernel at
 * D = 128) and exp2_poly_every (one exp2 pair in this many evaluated on the
 * FMA pipe, 0 = none).  A static string owned by the library; never NULL.
 * Lets a benchmark record which build it timed. */
LONGSPEC_HTA_API const char *longspec_hta_build_info(void);

/* Text of a status code; never NULL. */
LONGSPEC_HTA_API const char *longspec_hta_strerror(int code);

/* Split-KV chunk count the library uses for `dims` when num_splits = 0
 * (number of SMs of the current device enters the choice).  Returns a
 * negative status on invalid dims. */
LONGSPEC_HTA_API int longspec_hta_default_splits(const longspec_hta_dims *dims);

/* Split-KV chunking for a requested split count (0 = the default choice):
 * writes the number of chunks S actually used and the chunk length in keys
 * (a multiple of 128; chunk c covers prefix keys [c*C, (c+1)*C) clipped to
 * [0, L_b)).  Either output may be NULL. */
LONGSPEC_HTA_API int longspec_hta_chunking(const longspec_hta_dims *dims, int num_splits,
                                           int *num_splits_out, int *chunk_keys_out);

/* Workspace bytes needed by longspec_hta_verify(_ex) for `dims` and a split
 * count (0 = the default choice).  Holds the status word and the fp32 prefix
 * partials: B*Hq*T*S*(D+1)*4 bytes plus 256.  0 on invalid dims. */
LONGSPEC_HTA_API size_t longspec_hta_workspace_bytes(const longspec_hta_dims *dims, int num_splits);

/* Clears the workspace status word (asynchronously on `stream`).  Call once
 * after allocating a workspace; longspec_hta_get_status clears it again. */
LONGSPEC_HTA_API int longspec_hta_workspace_init(void *workspace, size_t workspace_bytes,
                                cudaStream_t stream);

/*
 * The verification attention of one layer: out and lse for every
 * (b, h, t).  Runs the split-KV prefix kernel (TMA + tcgen05, accumulators
 * in tensor memory) over prefix keys [0, L_b), then the tree kernel (ancestor
 * bitmask built from parent[] in shared memory, masked online softmax over
 * the tree keys) fused with the log-sum-exp merge of all partials.
 * Two kernel launches on `stream`.
 */
LONGSPEC_HTA_API int longspec_hta_verify(const longspec_hta_dims *dims,
                        const void *q, const void *k_prefix,
                        const void *v_prefix, const int32_t *prefix_len,
                        const void *k_tree, const void *v_tree,
                        const int32_t *parent, void *out, float *lse,
                        void *workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/* longspec_hta_verify with options (NULL = defaults). */
LONGSPEC_HTA_API int longspec_hta_verify_ex(const longspec_hta_dims *dims,
                           const void *q, const void *k_prefix,
                           const void *v_prefix, const int32_t *prefix_len,
                           const void *k_tree, const void *v_tree,
                           const int32_t *parent, void *out, float *lse,
                           void *workspace, size_t workspace_bytes,
                           const longspec_hta_options *opts,
                           cudaStream_t stream);

/*
 * longspec_hta_verify with no workspace argument, for callers that cannot
 * allocate device memory (a serving engine that reserves all device memory
 * at start-up and allows no later allocation, or a decode step in which a
 * cudaMalloc would synchronise the device).  The pages describe no such
 * entry point; it has no counterpart there.
 *   Scratch: a 16 MiB device array inside the library (status word and
 *   prefix split partials), held by every GPU that loads the library until
 *   the process exits.  The call picks the largest split count whose
 *   partials fit; a problem whose partials do not fit even with one split
 *   (B*Hq*T*(D+1)*4 bytes + 256 > 16 MiB) returns
 *   LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL and launches nothing.
 *   Set-up: the first call on each device, and the first call after the
 *   current context on that device changed (a device reset, or a
 *   driver-API context made current instead of the primary one), looks up
 *   the array's device address (cudaGetSymbolAddress) in the current
 *   context; make that first call before any stream capture.
 *   Sharing: every call on a device uses the same array.  Calls that can
 *   overlap on the GPU (different streams, or different host threads with no
 *   ordering between them) race on it and must be serialised by the caller.
 *   Device-detected problems (bad parent[], prefix_len out of range) show as
 *   NaN rows of out/lse; there is no status word to query.
 *   Allocation: calls no cudaMalloc/cudaFree or any allocating routine.
 */
LONGSPEC_HTA_API int longspec_hta_verify_noalloc(const longspec_hta_dims *dims,
                                const void *q, const void *k_prefix,
                                const void *v_prefix, const int32_t *prefix_len,
                                const void *k_tree, const void *v_tree,
                                const int32_t *parent, void *out, float *lse,
                                cudaStream_t stream);

/*
 * The split-KV chunking longspec_hta_verify_noalloc uses on a GPU with
 * num_sms SMs (host only, no device needed): the split count
 * longspec_hta_chunking would choose, lowered until the partials fit in the
 * library's 16 MiB scratch.  Writes the split count and the keys per chunk;
 * LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL when not even one split fits.  No
 * counterpart in the pages.
 */
LONGSPEC_HTA_API int longspec_hta_noalloc_chunking(const longspec_hta_dims *dims, int num_sms,
                                  int *num_splits_out, int *chunk_keys_out);

/* Device bytes of the staging arena longspec_hta_verify_host needs: room
 * for every input and output plus the workspace, each 256-byte aligned. */
LONGSPEC_HTA_API size_t longspec_hta_host_arena_bytes(const longspec_hta_dims *dims);

/*
 * End-to-end call on HOST buffers (same layouts, host pointers; pinned
 * memory gives asynchronous copies).  Copies the inputs into the caller's
 * device `arena` (longspec_hta_host_arena_bytes), runs longspec_hta_verify,
 * and copies out and lse back, all on `stream`; the host results are valid
 * after the stream is synchronised.  The status word lives in the arena and
 * is cleared by this call before the launch.
 */
LONGSPEC_HTA_API int longspec_hta_verify_host(const longspec_hta_dims *dims,
                             const void *q, const void *k_prefix,
                             const void *v_prefix, const int32_t *prefix_len,
                             const void *k_tree, const void *v_tree,
                             const int32_t *parent, void *out, float *lse,
                             void *arena, size_t arena_bytes,
                             cudaStream_t stream);

/*
 * Debug export of the tree mask: bits uint32 [B][T][ceil(T/32)], bit k of
 * word w of row i set iff node 32w+k is node i or an ancestor of i.  Same
 * device code as the tree kernel's shared-memory mask.  Bad parents are
 * reported through the status word of `workspace` (>= 256 bytes) and their
 * trees' rows are written as all ones.
 */
LONGSPEC_HTA_API int longspec_hta_tree_mask(const int32_t *parent, int B, int T, uint32_t *bits,
                           void *workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/*
 * Debug export of the tree partial alone: attention of every (b, h, t) over
 * its visible tree keys only.  o_tree fp32 [B][Hq][T][D] (normalised),
 * lse_tree fp32 [B][Hq][T] (natural log).  Same kernel as verify's tree pass.
 * Needs a workspace of >= 256 bytes for the status word.
 */
LONGSPEC_HTA_API int longspec_hta_tree_partial(const longspec_hta_dims *dims, const void *q,
                              const void *k_tree, const void *v_tree,
                              const int32_t *parent, float *o_tree,
                              float *lse_tree, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream);

/*
 * Debug export of the prefix split-KV partials alone.  o_part fp32
 * [B][Hq][T][S][D] (each normalised over its chunk), lse_part fp32
 * [B][Hq][T][S] (natural log; -inf for an empty chunk).  Chunk c covers
 * prefix keys [c*C, (c+1)*C) clipped to [0, L_b), C = chunk size the
 * library derives from L_cap and S (a multiple of 128).  num_splits 0 =
 * default.  Writes S to *num_splits_out if non-NULL.
 */
LONGSPEC_HTA_API int longspec_hta_prefix_partial(const longspec_hta_dims *dims, const void *q,
                                const void *k_prefix, const void *v_prefix,
                                const int32_t *prefix_len, float *o_part,
                                float *lse_part, int num_splits,
                                int prefix_kernel, int *num_splits_out,
                                void *workspace, size_t workspace_bytes,
                                cudaStream_t stream);

/* Attention of the query rows to the prefix alone: no tree keys, no mask.
 * This is the draft model's cross-attention into the target's KV cache in
 * LongSpec (LongSpec paper summary, "Summary": the draft attends to the
 * target model's KV cache), the prefix pass of verify followed by the same
 * exact lse merge of its split-KV partials, without the tree partial:
 *   out[b][h][t] = sum_{j < L_b} e^{s q.k_j - m} v_j / sum_{j < L_b} e^{s q.k_j - m},
 *   lse[b][h][t] = m + ln sum_{j < L_b} e^{s q.k_j - m}   (natural log).
 * dims->T is the number of query tokens per head (1 <= T <= 256); q, k_prefix,
 * v_prefix, prefix_len, out and lse have the layouts of longspec_hta_verify;
 * there is no k_tree, v_tree or parent.  A row with L_b = 0 sees no key:
 * its out is 0 and its lse is -inf.  workspace / options / errors: as
 * longspec_hta_verify_ex (longspec_hta_workspace_bytes gives the size). */
LONGSPEC_HTA_API int longspec_hta_prefix_attention(const longspec_hta_dims *dims, const void *q,
                                  const void *k_prefix, const void *v_prefix,
                                  const int32_t *prefix_len, void *out, float *lse,
                                  void *workspace, size_t workspace_bytes,
                                  const longspec_hta_options *opts, cudaStream_t stream);

/* longspec_hta_verify_ex and longspec_hta_prefix_attention with the prefix
 * K/V read from a paged cache (longspec_hta_paged_kv) instead of the
 * contiguous [B][Hkv][L_cap][D] arrays; every other argument, the result
 * and the error behaviour are the same.  The results equal those of the
 * contiguous call on the same keys bit for bit (same kernels, same split).
 * prefix_kernel LONGSPEC_HTA_PREFIX_SIMT returns
 * LONGSPEC_HTA_ERR_INVALID_OPTION.  Host
 * errors: NULL_POINTER / MISALIGNED for the cache and table pointers,
 * INVALID_DIMS for a block_size not in {16, 32, 64, 128}, num_blocks < 1,
 * max_blocks * block_size < L_cap or a cache over 2^31 rows. */
LONGSPEC_HTA_API int longspec_hta_verify_paged(const longspec_hta_dims *dims, const void *q,
                                const longspec_hta_paged_kv *kv, const int32_t *prefix_len,
                                const void *k_tree, const void *v_tree, const int32_t *parent,
                                void *out, float *lse, void *workspace, size_t workspace_bytes,
                                const longspec_hta_options *opts, cudaStream_t stream);
LONGSPEC_HTA_API int longspec_hta_prefix_attention_paged(const longspec_hta_dims *dims, const void *q,
                                const longspec_hta_paged_kv *kv, const int32_t *prefix_len,
                                void *out, float *lse, void *workspace, size_t workspace_bytes,
                                const longspec_hta_options *opts, cudaStream_t stream);

/* Greedy (temperature 0) acceptance of the speculated tree against the
 * target model's logits: the step after verification attention.  LongSpec
 * runs at temperature 0 (LongSpec README, "Inference": --temperature 0), so
 * the target's token after a position is the argmax of its logits there.
 * Node i of tree b is accepted when every node on its root path carries
 * the target's argmax token at that node's parent position:
 *   logits       bf16 [B][T+1][V], device: row 0 is the prefix end (judges
 *                the root-level nodes, parent -1), row 1+i the position
 *                after node i;
 *   draft_tokens int32 [B][T], parent int32 [B][T] (as in verify);
 *   accept_len   int32 [B]: depth of the deepest accepted node, 0 if none;
 *   path         int32 [B][T]: its root path, node ids from depth 1, then -1;
 *   bonus        int32 [B]: the target's argmax at the last accepted position
 *                (row 0 when nothing is accepted), the token emitted after
 *                the accepted ones.
 * Among equally deep accepted nodes the smallest id wins; argmax ties go to
 * the smallest token id; a NaN logit counts as -inf.  workspace: device, 16-byte
 * aligned, longspec_hta_accept_workspace_bytes bytes (status word first).
 * Errors: INVALID_DIMS (B, T, V < 1, B*(T+1) > 65535), T_TOO_LARGE,
 * NULL_POINTER, MISALIGNED (logits and workspace 16 bytes, the int32 arrays
 * 4 bytes), WORKSPACE_TOO_SMALL; a bad parent array gives accept_len 0 and
 * LONGSPEC_HTA_ERR_BAD_PARENT from longspec_hta_get_status. */
LONGSPEC_HTA_API size_t longspec_hta_accept_workspace_bytes(int B, int T, int V);
LONGSPEC_HTA_API int longspec_hta_accept_greedy(int B, int T, int V, const void *logits,
                                const int32_t *draft_tokens, const int32_t *parent,
                                int32_t *accept_len, int32_t *path, int32_t *bonus,
                                void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Sliding-window tree attention: the draft model's self-attention while it
 * drafts the tree.  LongSpec's draft model is one transformer block with
 * sliding-window self-attention over 512 positions (LongSpec paper summary,
 * "Summary"), so its own KV cache is a ring of W slots holding the last W
 * positions, position p at slot p mod W.  A query at position p sees the W
 * positions p - W + 1 .. p; a tree node at depth d (1 for parent -1) sits at
 * position L_b + d - 1, so it sees its d ancestors-or-self and the context
 * positions L_b + d - W .. L_b - 1 (clipped at 0):
 *   dims: B, Hq, Hkv, D, T as in verify; L_cap = W, the ring size, a
 *         multiple of 128 and > T (so a node's root path is in its window);
 *   q bf16 [B][Hq][T][D]; k_ring/v_ring bf16 [B][Hkv][W][D];
 *   prefix_len int32 [B]: the context length L_b >= 0 (it may exceed W);
 *   k_tree/v_tree bf16 [B][Hkv][T][D], parent int32 [B][T] as in verify;
 *   out bf16 [B][Hq][T][D], lse fp32 [B][Hq][T] (natural log);
 *   workspace: longspec_hta_window_workspace_bytes(dims) bytes, 16-byte
 *         aligned (status word first).
 * Ring slots no position of the window maps to are never read as keys
 * (they may hold anything).  Runs the tcgen05 prefix kernel over the window's
 * W/128 + 1 tiles (one chunk per row tile and KV head) and the tree pass +
 * merge.  Errors: as verify, plus
 * INVALID_DIMS for a W that is not a multiple of 128 or not above T; a
 * negative prefix_len gives PREFIX_LEN_RANGE and NaN rows. */
LONGSPEC_HTA_API size_t longspec_hta_window_workspace_bytes(const longspec_hta_dims *dims);
LONGSPEC_HTA_API int longspec_hta_window_verify(const longspec_hta_dims *dims, const void *q,
                                const void *k_ring, const void *v_ring, const int32_t *prefix_len,
                                const void *k_tree, const void *v_tree, const int32_t *parent,
                                void *out, float *lse, void *workspace, size_t workspace_bytes,
                                cudaStream_t stream);

/* Commit of the accepted path: after verification and acceptance, the
 * accepted tokens join the target's context, so their K/V rows (the tree
 * keys the verification pass used) are appended to the KV cache right after
 * the prefix and the prefix grows by the accepted length (LongSpec README,
 * "Introduction": the target model verifies the speculated tree and keeps
 * the accepted tokens; rejected branches are dropped).  For every sequence b
 * with L_b = prefix_len[b], n_b = accept_len[b] and every KV head h:
 *   cache_K[b][h][L_b + d] = k_tree[b][h][path[b][d]],  d < n_b (V alike),
 * then prefix_len[b] = L_b + n_b (in place, on the device).  Cache rows past
 * L_b + n_b are not touched.
 *   dims: B, Hkv, D, T, L_cap as in verify (Hq and scale only validated);
 *   k_prefix/v_prefix: the contiguous cache bf16 [B][Hkv][L_cap][D];
 *   kv: a paged cache (position p of sequence b is row p % block_size of
 *       block block_table[b][p / block_size]); the commit writes through
 *       kv->k_cache and kv->v_cache, and the table must already map every
 *       position below L_b + n_b;
 *   prefix_len int32 [B] (read, then advanced); k_tree/v_tree bf16
 *   [B][Hkv][T][D]; accept_len int32 [B] and path int32 [B][T] as written by
 *   longspec_hta_accept_greedy (device; may come from the previous kernel on
 *   the stream, no host synchronisation is needed);
 *   workspace: device, at least 256 bytes (the status word).
 * Host errors: NULL_POINTER, MISALIGNED (caches, tree K/V and workspace 16
 * bytes; the int32 arrays 4 bytes), INVALID_DIMS, UNSUPPORTED_D,
 * T_TOO_LARGE, WORKSPACE_TOO_SMALL.  Device errors leave the sequence
 * unchanged (no row written, prefix_len kept) and set the status word:
 * BAD_PATH (n_b outside [0, T] or a path entry outside [0, T)),
 * PREFIX_LEN_RANGE (L_b outside [0, L_cap] or L_b + n_b > L_cap), BAD_BLOCK. */
LONGSPEC_HTA_API int longspec_hta_commit(const longspec_hta_dims *dims, void *k_prefix, void *v_prefix,
                                int32_t *prefix_len, const void *k_tree, const void *v_tree,
                                const int32_t *accept_len, const int32_t *path, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream);
LONGSPEC_HTA_API int longspec_hta_commit_paged(const longspec_hta_dims *dims, const longspec_hta_paged_kv *kv,
                                int32_t *prefix_len, const void *k_tree, const void *v_tree,
                                const int32_t *accept_len, const int32_t *path, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream);

/* Synchronises `stream`, reads and clears the status word of `workspace`,
 * and returns LONGSPEC_HTA_OK or the first device-detected error. */
LONGSPEC_HTA_API int longspec_hta_get_status(void *workspace, cudaStream_t stream);

/* Self-test of failure detection (a test hook; the pages define no such
 * operation).  Launches one CTA on `stream` whose thread waits, with the
 * same bounded wait as every pipeline stage of the verification kernels,
 * on a barrier that nothing completes.  After the bound (about 2 s of SM
 * cycles) the wait gives up and sets the PIPELINE_TIMEOUT bit in the
 * status word of `workspace` (device memory, 16-byte aligned, at least
 * 256 bytes, e.g. a verification workspace), exactly as a stalled stage
 * would; the kernel then returns and the context stays usable.  Returns
 * LONGSPEC_HTA_OK once launched, NULL_POINTER / MISALIGNED /
 * UNSUPPORTED_DEVICE / CUDA otherwise; longspec_hta_get_status then
 * reports LONGSPEC_HTA_ERR_PIPELINE_TIMEOUT. */
LONGSPEC_HTA_API int longspec_hta_selftest_wait_timeout(void *workspace, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LONGSPEC_HTA_H */
