// tree_merge.cu -- tree pass of Hybrid Tree Attention fused with the
// log-sum-exp aggregation of all partials.
//
// LongSpec README, "Introduction" (hybrid attention aggregation: standard
// attention for the tree mask) and the LongSpec paper summary, "Summary"
// (the speculated tree gets its own kernel next to the prefix pass).
//
// One CTA = 8 warps for one (b, KV head) and up to 16 packed rows
// r = g*T + t of that head's query group.  The CTA
//   1. loads parent[b][:] into shared memory, checks parent[i] in [-1, i),
//   2. builds the ancestor-or-self bitmask of every node in shared memory by
//      pointer jumping (log2 T rounds: anc[i] |= anc[jump[i]],
//      jump[i] = jump[jump[i]]), so deep chains cost no more than bushy trees,
//   3. runs, one warp per row, the masked online softmax over the visible
//      tree keys only (the mask bits are walked, never the full T x T grid),
//   4. merges the tree partial with the S prefix split-KV partials by
//      log-sum-exp rescaling and writes out (bf16) and lse (fp32).
// Modes export the mask or the tree partial alone (debug entry points).
#include "hta_kernels.h"

namespace hta {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int D>
__device__ void tree_rows(const TreeMergeParams &p, const uint32_t (*anc)[kMaskWords],
                          int b, int kvh, bool bad_parent) {
    constexpr int DPL = D / 32;   // values per lane
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int G = p.Hq / p.Hkv, M = G * p.T, W = (p.T + 31) / 32;
    const float nan = __int_as_float(0x7fc00000);
    const int L = p.prefix_len ? p.prefix_len[b] : 0;
    const bool bad_len = (p.mode == kTreeModeMerge) && (L < 0 || L > p.L_cap);
    if (bad_len && threadIdx.x == 0 && blockIdx.x == 0)
        raise_status(p.status, kStatusPrefixLenRange);

    for (int rr = blockIdx.x * kTreeRowsPerCta + warp; rr < min(M, (blockIdx.x + 1) * kTreeRowsPerCta);
         rr += kWarps) {
        const int g = rr / p.T, t = rr % p.T, h = kvh * G + g;
        const size_t row = (static_cast<size_t>(b) * p.Hq + h) * p.T + t;
        const size_t kv_base = (static_cast<size_t>(b) * p.Hkv + kvh) * p.T;
        float acc[DPL];
        float m = -INFINITY, l = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[i] = 0.f;

        if (!bad_parent) {
            float qv[DPL];
            const __nv_bfloat16 *qr = p.q + row * D + lane * DPL;
#pragma unroll
            for (int i = 0; i < DPL; ++i) qv[i] = __bfloat162float(qr[i]);
            for (int w = 0; w < W; ++w) {
                uint32_t bits = anc[t][w];
                while (bits) {
                    const int j = w * 32 + (__ffs(bits) - 1);
                    bits &= bits - 1;
                    const __nv_bfloat16 *kr = p.k_tree + (kv_base + j) * D + lane * DPL;
                    const __nv_bfloat16 *vr = p.v_tree + (kv_base + j) * D + lane * DPL;
                    float dot = 0.f;
#pragma unroll
                    for (int i = 0; i < DPL; ++i) dot = fmaf(qv[i], __bfloat162float(kr[i]), dot);
                    const float x = warp_sum(dot) * p.scale_log2;
                    const float m_new = fmaxf(m, x);
                    const float a = ex2(m - m_new);      // m = -inf -> 0
                    const float pj = ex2(x - m_new);
                    l = l * a + pj;
#pragma unroll
                    for (int i = 0; i < DPL; ++i)
                        acc[i] = fmaf(pj, __bfloat162float(vr[i]), acc[i] * a);
                    m = m_new;
                }
            }
        }

        if (p.mode == kTreeModePartial) {
            // the tree partial alone: O_tree (normalised) and lse_tree (natural log)
            float *o = p.o_tree + row * D + lane * DPL;
            const float inv = bad_parent ? nan : 1.f / l;
#pragma unroll
            for (int i = 0; i < DPL; ++i) o[i] = acc[i] * inv;
            if (lane == 0) p.lse_tree[row] = bad_parent ? nan : (m + lg2(l)) * kLn2;
            continue;
        }

        // merge: the tree partial (m, l, acc in log2 units) with S prefix partials
        float out_v[DPL];
        float lse_out;
        if (bad_parent || bad_len) {
#pragma unroll
            for (int i = 0; i < DPL; ++i) out_v[i] = nan;
            lse_out = nan;
        } else {
            const float lse2_tree = m + lg2(l);
            const float *lp = p.lse_part + row * p.S;
            float mx = lse2_tree;
            bool has_nan = false;
            for (int s = 0; s < p.S; ++s) {
                const float v = lp[s];
                has_nan |= (v != v);
                mx = fmaxf(mx, v * kLog2e);
            }
            float wsum = ex2(lse2_tree - mx);
            const float wt = wsum / l;
#pragma unroll
            for (int i = 0; i < DPL; ++i) out_v[i] = acc[i] * wt;
            const float *op = p.o_part + row * static_cast<size_t>(p.S) * D + lane * DPL;
            for (int s = 0; s < p.S; ++s) {
                const float v = lp[s];
                if (v == -INFINITY) continue;
                const float w = ex2(v * kLog2e - mx);
                wsum += w;
                if constexpr (DPL == 4) {
                    const float4 o4 = *reinterpret_cast<const float4 *>(op + static_cast<size_t>(s) * D);
                    out_v[0] = fmaf(w, o4.x, out_v[0]);
                    out_v[1] = fmaf(w, o4.y, out_v[1]);
                    out_v[2] = fmaf(w, o4.z, out_v[2]);
                    out_v[3] = fmaf(w, o4.w, out_v[3]);
                } else {
                    const float2 o2 = *reinterpret_cast<const float2 *>(op + static_cast<size_t>(s) * D);
                    out_v[0] = fmaf(w, o2.x, out_v[0]);
                    out_v[1] = fmaf(w, o2.y, out_v[1]);
                }
            }
            const float inv = 1.f / wsum;
#pragma unroll
            for (int i = 0; i < DPL; ++i) out_v[i] = has_nan ? nan : out_v[i] * inv;
            lse_out = has_nan ? nan : (mx + lg2(wsum)) * kLn2;
        }
        __nv_bfloat16 *orow = p.out + row * D + lane * DPL;
        if constexpr (DPL == 4) {
            uint2 pk;
            pk.x = pack_bf16x2(out_v[0], out_v[1]);
            pk.y = pack_bf16x2(out_v[2], out_v[3]);
            *reinterpret_cast<uint2 *>(orow) = pk;
        } else {
            *reinterpret_cast<uint32_t *>(orow) = pack_bf16x2(out_v[0], out_v[1]);
        }
        if (lane == 0) p.lse[row] = lse_out;
    }
}

}  // namespace

// Ancestor-or-self mask of tree b into shared memory; returns true if the
// parent array is invalid (then the mask holds only the self bits).
__device__ bool build_tree_mask(const int32_t *parent_b, int T, int *s_jump,
                                uint32_t (*s_anc)[kMaskWords], int *s_flag) {
    const int i = threadIdx.x;   // T <= kTMax == blockDim.x
    const int W = (T + 31) / 32;
    if (i == 0) *s_flag = 0;
    __syncthreads();
    int jump = -1;
    uint32_t bits[kMaskWords];
#pragma unroll
    for (int w = 0; w < kMaskWords; ++w) bits[w] = 0;
    if (i < T) {
        jump = parent_b[i];
        if (jump < -1 || jump >= i) { *s_flag = 1; jump = -1; }
        bits[i / 32] = 1u << (i % 32);
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w) if (w < W) s_anc[i][w] = bits[w];
        s_jump[i] = jump;
    }
    __syncthreads();
    const bool bad = *s_flag != 0;
    // pointer jumping: anc[i] covers the path from i up to (not including)
    // jump[i]; each round doubles the covered length.
    while (__syncthreads_or(!bad && i < T && jump >= 0)) {
        int nj = -1;
        if (!bad && i < T && jump >= 0) {
#pragma unroll
            for (int w = 0; w < kMaskWords; ++w) if (w < W) bits[w] |= s_anc[jump][w];
            nj = s_jump[jump];
        }
        __syncthreads();
        if (!bad && i < T && jump >= 0) {
#pragma unroll
            for (int w = 0; w < kMaskWords; ++w) if (w < W) s_anc[i][w] = bits[w];
            s_jump[i] = nj;
            jump = nj;
        }
    }
    return bad;
}

__global__ void __launch_bounds__(kThreads)
tree_merge_kernel(TreeMergeParams p) {
    __shared__ int s_jump[kTMax];
    __shared__ uint32_t s_anc[kTMax][kMaskWords];
    __shared__ int s_flag;
    const int b = blockIdx.z, kvh = blockIdx.y;
    const bool bad = build_tree_mask(p.parent + static_cast<size_t>(b) * p.T, p.T, s_jump, s_anc, &s_flag);
    if (bad && threadIdx.x == 0 && blockIdx.x == 0 && kvh == 0)
        raise_status(p.status, kStatusBadParent);

    if (p.mode == kTreeModeMask) {
        const int W = (p.T + 31) / 32;
        for (int idx = threadIdx.x; idx < p.T * W; idx += blockDim.x) {
            const int i = idx / W, w = idx % W;
            p.mask_out[(static_cast<size_t>(b) * p.T + i) * W + w] = bad ? 0xffffffffu : s_anc[i][w];
        }
        return;
    }
    if (p.D == 128) tree_rows<128>(p, s_anc, b, kvh, bad);
    else tree_rows<64>(p, s_anc, b, kvh, bad);
}

cudaError_t launch_tree_merge(const TreeMergeParams &p, cudaStream_t stream) {
    dim3 grid;
    if (p.mode == kTreeModeMask) {
        grid = dim3(1, 1, p.B);
    } else {
        const int M = (p.Hq / p.Hkv) * p.T;
        grid = dim3((M + kTreeRowsPerCta - 1) / kTreeRowsPerCta, p.Hkv, p.B);
    }
    tree_merge_kernel<<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace hta
