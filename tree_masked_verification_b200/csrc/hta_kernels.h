// hta_kernels.h -- parameter blocks and launchers of the Hybrid Tree
// Attention kernels (internal to liblongspec_hta.so).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hta_common.cuh"

// Build-time tuning knobs of the tcgen05 prefix kernel (defaults = the
// measured best on B200; set with -D at build time, reported by
// longspec_hta_build_info):
//   HTA_KV_STAGES_D128   depth of the K and V rings at D = 128 (2 or 3; four
//                        stages of 32 KB each do not fit beside Q)
//   HTA_EXP2_POLY_EVERY  one exp2 pair in this many on the FMA pipe (0: all
//                        on the exp2 unit; 2, 4, 8 or 16)
#ifndef HTA_KV_STAGES_D128
#define HTA_KV_STAGES_D128 3
#endif
#ifndef HTA_EXP2_POLY_EVERY
#define HTA_EXP2_POLY_EVERY 4
#endif
static_assert(HTA_KV_STAGES_D128 == 2 || HTA_KV_STAGES_D128 == 3, "K/V ring depth at D = 128");
static_assert(HTA_EXP2_POLY_EVERY == 0 || HTA_EXP2_POLY_EVERY == 2 || HTA_EXP2_POLY_EVERY == 4 ||
              HTA_EXP2_POLY_EVERY == 8 || HTA_EXP2_POLY_EVERY == 16, "exp2 share on the FMA pipe");

namespace hta {

constexpr int kTreeRowsPerCta = 8;    // one warp per packed row
constexpr int kKeyTile = 128;   // keys per prefix tile; chunk sizes are multiples of it
constexpr int kMaxSplits = 64;  // prefix split-KV chunks per (b, KV head), at most

// Merge: tree pass + lse merge with the prefix partials.  PrefixOnly: the
// merge of the prefix partials alone (no tree keys; q rows attend to the
// prefix only).  Partial / Mask: debug exports of the tree pass.
enum TreeMode : int { kTreeModeMerge = 0, kTreeModePartial = 1, kTreeModeMask = 2,
                      kTreeModePrefixOnly = 3 };

struct TreeMergeParams {
    int B, Hq, Hkv, D, T, L_cap, S;
    float scale_log2;                 // softmax scale * log2(e)
    int mode;                         // TreeMode
    const __nv_bfloat16 *q, *k_tree, *v_tree;
    const int32_t *parent, *prefix_len;
    const float *o_part, *lse_part;   // [rows][S][D], [rows][S] (natural log)
    __nv_bfloat16 *out;
    float *lse;
    float *o_tree, *lse_tree;         // kTreeModePartial outputs
    uint32_t *mask_out;               // kTreeModeMask output [B][T][ceil(T/32)]
    uint32_t *status;
    int window;                       // > 0: sliding-window call, prefix_len may exceed L_cap
};

// Prefix split-KV partials.  Rows of one (b, KV head) are the packed query
// group r = g*T + t (g < G), contiguous in q; global row index
// (b*Hkv + kvh)*M + r equals (b*Hq + h)*T + t.
struct PrefixParams {
    int B, Hq, Hkv, D, T, L_cap;
    int G, M, m_tiles;                // M = G*T, m_tiles = ceil(M / 128)
    int S, chunk_tiles;               // split c covers keys [c, c+1) * chunk_tiles * 128
    float scale_log2;
    const __nv_bfloat16 *q, *k_prefix, *v_prefix;   // (SIMT kernel reads these directly)
    const int32_t *prefix_len;
    float *o_part, *lse_part;         // [rows][S][D], [rows][S]
    uint32_t *status;
    // Paged prefix K/V (tcgen05 kernel only): null block_table = contiguous
    // [B][Hkv][L_cap][D]; else the caches are [num_blocks][Hkv][block_size][D]
    // and the tensor maps' boxes are block_size rows high.
    const int32_t *block_table;       // [B][max_blocks]
    int block_size, max_blocks, num_blocks;
    // Sliding window (tcgen05 kernel only): window > 0 = the ring size W
    // (= L_cap, a multiple of 128, > T); context position p sits at slot
    // p mod W; a node at depth d sees positions [L_b + d - W, L_b).  The
    // chunks cover the W/128 + 1 tiles from the one holding L_b - W.
    int window;
    const int32_t *parent;            // [B][T], for the depths (window only)
};

// Greedy (temperature-0) acceptance of a speculated tree.  logits bf16
// [B][T+1][V]: row 0 = the prefix end, row 1+i = the position after node i.
struct AcceptParams {
    int B, T, V;
    int n_slices, slice;              // argmax slices per row, elements per slice (multiple of 8)
    const __nv_bfloat16 *logits;
    const int32_t *draft_tokens, *parent;   // [B][T]
    float *part_v;                    // [B*(T+1)][n_slices] slice maxima
    int *part_i;                      // [B*(T+1)][n_slices] their first indices
    int32_t *accept_len, *path, *bonus;     // [B], [B][T], [B]
    uint32_t *status;
};
cudaError_t launch_accept(const AcceptParams &p, cudaStream_t stream);

// Append the accepted path's tree K/V to the cache; prefix_len advances in place.
struct CommitParams {
    int B, Hkv, D, T, L_cap;
    __nv_bfloat16 *k_cache, *v_cache;          // [B][Hkv][L_cap][D], or paged [num_blocks][Hkv][block_size][D]
    const int32_t *block_table;                // [B][max_blocks], nullptr for a contiguous cache
    int block_size, max_blocks, num_blocks;
    int32_t *prefix_len;                       // [B], read and advanced
    const __nv_bfloat16 *k_tree, *v_tree;      // [B][Hkv][T][D]
    const int32_t *accept_len, *path;          // [B], [B][T]
    uint32_t *status;
};
cudaError_t launch_commit(const CommitParams &p, cudaStream_t stream);
cudaError_t launch_tree_merge(const TreeMergeParams &p, cudaStream_t stream);
// One bounded wait that is left to run out; sets kStatusPipelineTimeout.
cudaError_t launch_wait_timeout_selftest(uint32_t *status, cudaStream_t stream);
cudaError_t launch_prefix_simt(const PrefixParams &p, cudaStream_t stream);
// Tensor maps: q as [B*Hq*T][D], k/v as [B*Hkv*L_cap][D], box 64 x 128, 128B swizzle.
cudaError_t launch_prefix_tc(const PrefixParams &p, const CUtensorMap &tm_q,
                             const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                             cudaStream_t stream);

}  // namespace hta
