// tree_merge.cu -- tree pass of Hybrid Tree Attention fused with the
// log-sum-exp aggregation of all partials.
//
// LongSpec README, "Introduction" (hybrid attention aggregation: standard
// attention for the tree mask) and the LongSpec paper summary, "Summary"
// (the speculated tree gets its own kernel next to the prefix pass).
//
// One CTA = 8 warps for one (b, KV head) and up to 16 packed rows
// r = g*T + t of that head's query group.  The CTA
//   0. stages that head's tree K and V rows in shared memory,
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
                          const __nv_bfloat16 *s_k, const __nv_bfloat16 *s_v, int b, int kvh,
                          bool bad_parent) {
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
                    const __nv_bfloat16 *kr = s_k + j * D + lane * DPL;
                    const __nv_bfloat16 *vr = s_v + j * D + lane * DPL;
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

        // merge: the tree partial (m, l, acc; log2 units) with S prefix partials
        float out_v[DPL];
        float lse_out;
        if (bad_parent || bad_len) {
#pragma unroll
            for (int i = 0; i < DPL; ++i) out_v[i] = nan;
            lse_out = nan;
        } else {
            const float lse2_tree = m + lg2(l);
            const float *lp = p.lse_part + row * p.S;
            // every lane loads up to two partials' lse at once (S <= 64)
            const float v0 = lane < p.S ? lp[lane] * kLog2e : -INFINITY;
            const float v1 = lane + 32 < p.S ? lp[lane + 32] * kLog2e : -INFINITY;
            const bool has_nan = __any_sync(0xffffffffu, (v0 != v0) || (v1 != v1));
            float mx = fmaxf(fmaxf(v0, v1), lse2_tree);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float w0 = ex2(v0 - mx), w1 = ex2(v1 - mx);   // -inf -> 0
            const float wt = ex2(lse2_tree - mx);
            const float wsum = warp_sum(w0 + w1) + wt;
            const float ft = wt / l;
#pragma unroll
            for (int i = 0; i < DPL; ++i) out_v[i] = acc[i] * ft;
            const float *op = p.o_part + row * static_cast<size_t>(p.S) * D + lane * DPL;
            for (int s0 = 0; s0 < p.S; s0 += 8) {
                // issue up to 8 partial loads before using any of them
                float ld[8][DPL];
                float ws[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int s = s0 + u;
                    ws[u] = __shfl_sync(0xffffffffu, s < 32 ? w0 : w1, s & 31);
                    const bool live = s < p.S && ws[u] > 0.f;
                    if constexpr (DPL == 4) {
                        const float4 v = live ? *reinterpret_cast<const float4 *>(op + static_cast<size_t>(s) * D)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
                        ld[u][0] = v.x; ld[u][1] = v.y; ld[u][2] = v.z; ld[u][3] = v.w;
                    } else {
                        const float2 v = live ? *reinterpret_cast<const float2 *>(op + static_cast<size_t>(s) * D)
                                              : make_float2(0.f, 0.f);
                        ld[u][0] = v.x; ld[u][1] = v.y;
                    }
                    if (!live) ws[u] = 0.f;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u)
#pragma unroll
                    for (int i = 0; i < DPL; ++i) out_v[i] = fmaf(ws[u], ld[u][i], out_v[i]);
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
    extern __shared__ uint4 s_tree[];   // tree K rows [T][D] then tree V rows [T][D] (bf16)
    const int b = blockIdx.z, kvh = blockIdx.y;
    if (p.mode != kTreeModeMask) {
        // stage this head's tree keys and values once (coalesced 16-byte
        // loads); the __syncthreads of the mask build below orders them
        const int n16 = p.T * p.D / 8;
        const size_t base = (static_cast<size_t>(b) * p.Hkv + kvh) * p.T * p.D / 8;
        const uint4 *kg = reinterpret_cast<const uint4 *>(p.k_tree) + base;
        const uint4 *vg = reinterpret_cast<const uint4 *>(p.v_tree) + base;
        for (int i = threadIdx.x; i < n16; i += blockDim.x) {
            s_tree[i] = kg[i];
            s_tree[n16 + i] = vg[i];
        }
    }
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
    const __nv_bfloat16 *s_k = reinterpret_cast<const __nv_bfloat16 *>(s_tree);
    const __nv_bfloat16 *s_v = s_k + p.T * p.D;
    if (p.D == 128) tree_rows<128>(p, s_anc, s_k, s_v, b, kvh, bad);
    else tree_rows<64>(p, s_anc, s_k, s_v, b, kvh, bad);
}

cudaError_t launch_tree_merge(const TreeMergeParams &p, cudaStream_t stream) {
    dim3 grid;
    size_t smem = 0;
    if (p.mode == kTreeModeMask) {
        grid = dim3(1, 1, p.B);
    } else {
        const int M = (p.Hq / p.Hkv) * p.T;
        grid = dim3((M + kTreeRowsPerCta - 1) / kTreeRowsPerCta, p.Hkv, p.B);
        smem = static_cast<size_t>(p.T) * p.D * 2 * 2;
        constexpr int kMaxDev = 64;
        static bool attr_set[kMaxDev] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (smem > 48 * 1024 && (dev < 0 || dev >= kMaxDev || !attr_set[dev])) {
            e = cudaFuncSetAttribute(tree_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(kTMax) * 128 * 2 * 2);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < kMaxDev) attr_set[dev] = true;
        }
    }
    tree_merge_kernel<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace hta
