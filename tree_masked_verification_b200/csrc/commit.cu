// commit.cu -- append the accepted path's tree K/V to the prefix cache.
//
// After verification (LongSpec README, "Introduction": the target model
// checks the speculated tree) and greedy acceptance, the accepted tokens
// become part of the target's context: their K/V rows, computed by the
// verification forward pass as tree keys, move into the KV cache right
// after the sequence's prefix, and the prefix grows by the accepted length.
// The rejected branches are dropped (nothing is written for them).
//
// One CTA per sequence b (so that the in-place prefix_len update needs no
// grid-wide order): it reads L_b, the accepted length n_b and the path,
// checks them, then copies K and V of every KV head for depth d < n_b from
// tree row path[b][d] to cache position L_b + d in 16-byte pieces, up to
// eight in flight per thread, and finally writes prefix_len[b] = L_b + n_b.
// The cache is contiguous [B][Hkv][L_cap][D] or paged
// [num_blocks][Hkv][block_size][D] through a block table.
#include "hta_kernels.h"

namespace hta {

namespace {

constexpr int kCommitThreads = 256;

__global__ void __launch_bounds__(kCommitThreads)
commit_kernel(CommitParams p) {
    // the accepted lengths and paths come from the previous kernel on the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ int s_path[kTMax];
    __shared__ int s_blk[kTMax];
    __shared__ int s_ok;
    const int b = blockIdx.x, T = p.T;
    const int L = p.prefix_len[b];
    const int n = p.accept_len[b];
    if (threadIdx.x == 0) s_ok = 1;
    __syncthreads();
    if (threadIdx.x == 0) {
        if (n < 0 || n > T) {
            raise_status(p.status, kStatusBadPath);
            s_ok = 0;
        } else if (L < 0 || L > p.L_cap || n > p.L_cap - L) {
            raise_status(p.status, kStatusPrefixLenRange);
            s_ok = 0;
        }
    }
    __syncthreads();
    if (!s_ok) return;
    for (int d = threadIdx.x; d < n; d += blockDim.x) {
        const int node = p.path[static_cast<size_t>(b) * T + d];
        if (node < 0 || node >= T) {
            raise_status(p.status, kStatusBadPath);
            s_ok = 0;
        }
        s_path[d] = node;
        if (p.block_table) {
            const int pos = L + d;
            const int blk = p.block_table[static_cast<size_t>(b) * p.max_blocks + pos / p.block_size];
            if (blk < 0 || blk >= p.num_blocks) {
                raise_status(p.status, kStatusBadBlock);
                s_ok = 0;
            }
            s_blk[d] = blk;
        }
    }
    __syncthreads();
    if (!s_ok) return;   // the sequence is left as it was

    // piece k of (kv, h, d, c): kv 0 = K, 1 = V; c = 16-byte column piece
    const int pieces_row = p.D / 8;
    const int total = 2 * p.Hkv * n * pieces_row;
    for (int k0 = threadIdx.x; k0 < total; k0 += 8 * kCommitThreads) {
        uint4 v[8];
        size_t dst[8];
        bool is_v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int k = k0 + u * kCommitThreads;
            if (k < total) {
                const int c = k % pieces_row;
                const int rest = k / pieces_row;
                const int d = rest % n;
                const int hk = rest / n;           // kv * Hkv + h
                const int h = hk % p.Hkv, kv = hk / p.Hkv;
                const __nv_bfloat16 *src = (kv ? p.v_tree : p.k_tree) +
                    ((static_cast<size_t>(b) * p.Hkv + h) * T + s_path[d]) * p.D;
                v[u] = __ldg(reinterpret_cast<const uint4 *>(src) + c);
                size_t row;
                if (p.block_table) {
                    const int pos = L + d;
                    row = (static_cast<size_t>(s_blk[d]) * p.Hkv + h) * p.block_size + pos % p.block_size;
                } else {
                    row = (static_cast<size_t>(b) * p.Hkv + h) * p.L_cap + (L + d);
                }
                dst[u] = row * pieces_row + c;
                is_v[u] = kv != 0;
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int k = k0 + u * kCommitThreads;
            if (k < total)
                reinterpret_cast<uint4 *>(is_v[u] ? p.v_cache : p.k_cache)[dst[u]] = v[u];
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __syncthreads();   // every thread has read L before it changes
    if (threadIdx.x == 0) p.prefix_len[b] = L + n;
}

}  // namespace

cudaError_t launch_commit(const CommitParams &p, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = stream;
    cfg.gridDim = dim3(p.B);
    cfg.blockDim = dim3(kCommitThreads);
    return cudaLaunchKernelEx(&cfg, commit_kernel, p);
}

}  // namespace hta
