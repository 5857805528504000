// tree_merge.cu -- tree pass of Hybrid Tree Attention fused with the
// log-sum-exp aggregation of all partials.
//
// LongSpec README, "Introduction" (hybrid attention aggregation: standard
// attention for the tree mask) and the LongSpec paper summary, "Summary"
// (the speculated tree gets its own kernel next to the prefix pass).
//
// One CTA = 8 warps = 8 packed rows r = g*T + t of one (b, KV head).  The CTA
//   1. loads parent[b][:] into shared memory, checks parent[i] in [-1, i),
//   2. builds the ancestor-or-self bitmask of every node in shared memory by
//      pointer jumping (log2 T rounds: anc[i] |= anc[jump[i]],
//      jump[i] = jump[jump[i]]), so deep chains cost no more than bushy trees,
//   3. runs, one warp per row, the online softmax over the visible tree keys
//      only (the mask bits are walked, never the full T x T grid), fetching
//      up to 4 visible keys' K and V rows at once,
//   4. waits for the prefix kernel (programmatic dependent launch: steps 1-3
//      overlap the prefix kernel's tail) and merges the tree partial with the
//      S split-KV partials by log-sum-exp rescaling, writing out (bf16) and
//      lse (fp32).
// Modes export the mask or the tree partial alone (debug entry points).
#include "hta_kernels.h"

namespace hta {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int D>
__device__ void tree_row(const TreeMergeParams &p, const uint32_t (*anc)[kMaskWords], int b,
                         int kvh, int rr, bool bad_parent) {
    constexpr int DPL = D / 32;   // values per lane
    constexpr int KB = 4;         // visible keys fetched at once
    const int lane = threadIdx.x % 32;
    const int G = p.Hq / p.Hkv, W = (p.T + 31) / 32;
    const float nan = __int_as_float(0x7fc00000);
    const int g = rr / p.T, t = rr % p.T, h = kvh * G + g;
    const size_t row = (static_cast<size_t>(b) * p.Hq + h) * p.T + t;
    const size_t kv_base = (static_cast<size_t>(b) * p.Hkv + kvh) * p.T;
    float acc[DPL];
    float m = -INFINITY, l = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] = 0.f;

    if (!bad_parent && p.mode != kTreeModePrefixOnly) {
        float qv[DPL];
        const __nv_bfloat16 *qr = p.q + row * D + lane * DPL;
#pragma unroll
        for (int i = 0; i < DPL; ++i) qv[i] = __bfloat162float(qr[i]);
        int w = 0;
        uint32_t bits = anc[t][0];
        for (;;) {
            int idx[KB];
            int n = 0;
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                while (bits == 0 && w + 1 < W) bits = anc[t][++w];
                idx[u] = bits ? w * 32 + (__ffs(bits) - 1) : -1;
                if (bits) { bits &= bits - 1; ++n; }
            }
            if (n == 0) break;
            // all K and V loads of the batch first, then the arithmetic
            float kf[KB][DPL], vf[KB][DPL];
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                const int j = idx[u] < 0 ? idx[0] : idx[u];
                // a key row is D contiguous bf16: one vector load per lane,
                // the warp reading the row as one coalesced 2*D-byte access
                const __nv_bfloat16 *kr = p.k_tree + (kv_base + j) * D + lane * DPL;
                const __nv_bfloat16 *vr = p.v_tree + (kv_base + j) * D + lane * DPL;
                if constexpr (DPL == 4) {
                    const uint2 kk = *reinterpret_cast<const uint2 *>(kr);
                    const uint2 vv = *reinterpret_cast<const uint2 *>(vr);
                    kf[u][0] = bf16_lo(kk.x); kf[u][1] = bf16_hi(kk.x);
                    kf[u][2] = bf16_lo(kk.y); kf[u][3] = bf16_hi(kk.y);
                    vf[u][0] = bf16_lo(vv.x); vf[u][1] = bf16_hi(vv.x);
                    vf[u][2] = bf16_lo(vv.y); vf[u][3] = bf16_hi(vv.y);
                } else {
                    const uint32_t kk = *reinterpret_cast<const uint32_t *>(kr);
                    const uint32_t vv = *reinterpret_cast<const uint32_t *>(vr);
                    kf[u][0] = bf16_lo(kk); kf[u][1] = bf16_hi(kk);
                    vf[u][0] = bf16_lo(vv); vf[u][1] = bf16_hi(vv);
                }
            }
            float x[KB];
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                float dot = 0.f;
#pragma unroll
                for (int i = 0; i < DPL; ++i) dot = fmaf(qv[i], kf[u][i], dot);
                x[u] = dot;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int u = 0; u < KB; ++u) x[u] += __shfl_xor_sync(0xffffffffu, x[u], o);
            float mb = -INFINITY;
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                x[u] = idx[u] < 0 ? -INFINITY : x[u] * p.scale_log2;
                mb = fmaxf(mb, x[u]);
            }
            const float m_new = fmaxf(m, mb);
            const float a = ex2(m - m_new);       // m = -inf -> 0
            l *= a;
#pragma unroll
            for (int i = 0; i < DPL; ++i) acc[i] *= a;
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                const float pj = ex2(x[u] - m_new);   // -inf -> 0
                l += pj;
#pragma unroll
                for (int i = 0; i < DPL; ++i) acc[i] = fmaf(pj, vf[u][i], acc[i]);
            }
            m = m_new;
            if (n < KB) break;
        }
    }

    if (p.mode == kTreeModePartial) {
        // the tree partial alone: O_tree (normalised) and lse_tree (natural log)
        float *o = p.o_tree + row * D + lane * DPL;
        const float inv = bad_parent ? nan : 1.f / l;
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[i] = acc[i] * inv;
        if (lane == 0) p.lse_tree[row] = bad_parent ? nan : (m + lg2(l)) * kLn2;
        return;
    }

    // merge: the tree partial (m, l, acc; log2 units) with S prefix partials.
    // prefix_len is an input of the call, like q and the tree K/V above:
    // read before the wait, so the partials' loads follow it directly.
    const int L = p.prefix_len[b];
    grid_dependency_wait();   // the prefix kernel's partials are complete and visible
    // The next kernel on the stream (the next call's prefix pass) may be
    // scheduled now: it waits for this grid before it reads anything.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const bool bad_len = L < 0 || (p.window == 0 && L > p.L_cap);
    if (bad_len && lane == 0 && rr == 0) raise_status(p.status, kStatusPrefixLenRange);
    float out_v[DPL];
    float lse_out;
    if (bad_parent || bad_len) {
#pragma unroll
        for (int i = 0; i < DPL; ++i) out_v[i] = nan;
        lse_out = nan;
    } else {
        const float lse2_tree = m + lg2(l);
        const float *lp = p.lse_part + row * p.S;
        const float *op = p.o_part + row * static_cast<size_t>(p.S) * D + lane * DPL;
        // the lse of every partial and the first 8 partial rows are loaded in
        // one round: the O loads do not wait for the weights (a partial with
        // weight 0 is dropped by a select below, so a slot a chunk past L_b
        // never wrote cannot leak in, whatever it holds)
        float ld[8][DPL];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if constexpr (DPL == 4) {
                const float4 v = u < p.S ? *reinterpret_cast<const float4 *>(op + static_cast<size_t>(u) * D)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                ld[u][0] = v.x; ld[u][1] = v.y; ld[u][2] = v.z; ld[u][3] = v.w;
            } else {
                const float2 v = u < p.S ? *reinterpret_cast<const float2 *>(op + static_cast<size_t>(u) * D)
                                         : make_float2(0.f, 0.f);
                ld[u][0] = v.x; ld[u][1] = v.y;
            }
        }
        // every lane loads up to two partials' lse at once (S <= 64)
        const float v0 = lane < p.S ? lp[lane] * kLog2e : -INFINITY;
        const float v1 = lane + 32 < p.S ? lp[lane + 32] * kLog2e : -INFINITY;
        const bool has_nan = __any_sync(0xffffffffu, (v0 != v0) || (v1 != v1));
        float mx = fmaxf(fmaxf(v0, v1), lse2_tree);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float w0 = ex2(v0 - mx), w1 = ex2(v1 - mx);   // -inf -> 0
        const float wt = ex2(lse2_tree - mx);
        float wsum = w0 + w1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
        wsum += wt;
        const float ft = l > 0.f ? wt / l : 0.f;   // no tree keys: weight 0
#pragma unroll
        for (int i = 0; i < DPL; ++i) out_v[i] = acc[i] * ft;
        for (int s0 = 0; s0 < p.S; s0 += 8) {
            if (s0 > 0) {   // partials 8.. (more than 8 splits): one more round per 8
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int s = s0 + u;
                    if constexpr (DPL == 4) {
                        const float4 v = s < p.S ? *reinterpret_cast<const float4 *>(op + static_cast<size_t>(s) * D)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
                        ld[u][0] = v.x; ld[u][1] = v.y; ld[u][2] = v.z; ld[u][3] = v.w;
                    } else {
                        const float2 v = s < p.S ? *reinterpret_cast<const float2 *>(op + static_cast<size_t>(s) * D)
                                                 : make_float2(0.f, 0.f);
                        ld[u][0] = v.x; ld[u][1] = v.y;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int s = s0 + u;
                const float ws = __shfl_sync(0xffffffffu, s < 32 ? w0 : w1, s & 31);
                const bool use = s < p.S && ws > 0.f;
#pragma unroll
                for (int i = 0; i < DPL; ++i) out_v[i] = use ? fmaf(ws, ld[u][i], out_v[i]) : out_v[i];
            }
        }
        const float inv = 1.f / wsum;
        const bool empty = mx == -INFINITY;   // no visible key at all (prefix-only, L_b = 0)
#pragma unroll
        for (int i = 0; i < DPL; ++i) out_v[i] = has_nan ? nan : empty ? 0.f : out_v[i] * inv;
        lse_out = has_nan ? nan : empty ? -INFINITY : (mx + lg2(wsum)) * kLn2;
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

// At most 64 registers (four CTAs per SM): the kernel is latency-bound, so
// more resident warps pay more than deeper batches of key loads.
__global__ void __launch_bounds__(kThreads, 4)
tree_merge_kernel(TreeMergeParams p) {
    __shared__ int s_jump[kTMax];
    __shared__ uint32_t s_anc[kTMax][kMaskWords];
    __shared__ int s_flag;
    const int b = blockIdx.z, kvh = blockIdx.y;
    // no tree keys in the prefix-only merge: no parent array, no mask
    const bool bad = p.mode == kTreeModePrefixOnly
                         ? false
                         : build_tree_mask(p.parent + static_cast<size_t>(b) * p.T, p.T, s_jump, s_anc, &s_flag);
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
    const int rr = blockIdx.x * kTreeRowsPerCta + threadIdx.x / 32;
    if (rr >= (p.Hq / p.Hkv) * p.T) return;
    if (p.D == 128) tree_row<128>(p, s_anc, b, kvh, rr, bad);
    else tree_row<64>(p, s_anc, b, kvh, rr, bad);
}

// ------------------------------------------------------- greedy acceptance
// Temperature-0 verification of the speculated tree against the target's
// logits: node i is accepted when every node on its root path carries the
// target's argmax token at that node's parent position; the deepest accepted
// chain (smallest id among equally deep nodes) and the target's argmax after
// it are the output.  Argmax ties go to the smallest token id; a NaN logit
// never wins.

namespace {

struct ArgBest {
    float v;
    int i;
};

// (v, i) beats (bv, bi): larger value, or the same value at a smaller index;
// a NaN counts as -inf (fmaxf returns the non-NaN operand)
__device__ __forceinline__ void arg_take(ArgBest &b, float v, int i) {
    v = fmaxf(v, -INFINITY);
    if (v > b.v || (v == b.v && i < b.i)) { b.v = v; b.i = i; }
}

constexpr int kArgThreads = 256;

// The larger of each bf16 pair (max.bf16x2: a NaN loses to a number).
__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Largest of the 8 bf16 values of a 16-byte chunk, as fp32 (NaN only if all
// 8 are NaN).
__device__ __forceinline__ float chunk_max8(uint4 u) {
    const uint32_t m = max_bf16x2(max_bf16x2(u.x, u.y), max_bf16x2(u.z, u.w));
    return fmaxf(bf16_lo(m), bf16_hi(m));
}

// Position (0..7) of the first of the 8 values of `u` equal to `v`
// (8 if none).
__device__ __forceinline__ int first_equal8(uint4 u, float v) {
    int e = 8;
    e = (bf16_hi(u.w) == v) ? 7 : e; e = (bf16_lo(u.w) == v) ? 6 : e;
    e = (bf16_hi(u.z) == v) ? 5 : e; e = (bf16_lo(u.z) == v) ? 4 : e;
    e = (bf16_hi(u.y) == v) ? 3 : e; e = (bf16_lo(u.y) == v) ? 2 : e;
    e = (bf16_hi(u.x) == v) ? 1 : e; e = (bf16_lo(u.x) == v) ? 0 : e;
    return e;
}

}  // namespace

// Slice `blockIdx.x` of row `blockIdx.y` of logits [rows][V] (bf16): its
// (max, first index) into part[row][slice].  Slices are `slice` elements
// long (a multiple of 8); rows whose start is 16-byte aligned are read with
// 16-byte loads, up to eight in flight per thread.
__global__ void __launch_bounds__(kArgThreads)
argmax_slices_kernel(const __nv_bfloat16 *logits, int V, int slice, float *part_v, int *part_i) {
    // the logits may come from the previous kernel on the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const size_t row = blockIdx.y;
    const int s = blockIdx.x, n_slices = gridDim.x;
    const int lo = s * slice, hi = min(V, lo + slice);
    const __nv_bfloat16 *x = logits + row * static_cast<size_t>(V);
    ArgBest b{-INFINITY, INT_MAX};
    if ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
        const uint4 *xv = reinterpret_cast<const uint4 *>(x);
        const int c_lo = lo / 8, c_hi = hi / 8;            // whole 8-element chunks
        // Up to eight 16-byte loads in flight per thread, then: the max of
        // each chunk (packed bf16 max), the batch max, and only where it
        // beats the best so far the first chunk and element holding it.  A
        // batch's indices grow with k and lie above every earlier batch's,
        // so the first match is the smallest index.  A batch holding only
        // NaN and -inf (all count as -inf) offers its first element.
        for (int c = c_lo + threadIdx.x; c < c_hi; c += 8 * kArgThreads) {
            uint4 u[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                u[k] = c + k * kArgThreads < c_hi ? __ldcs(xv + c + k * kArgThreads) : make_uint4(0u, 0u, 0u, 0u);
            float cm[8];
            float tm = -INFINITY;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                cm[k] = c + k * kArgThreads < c_hi ? chunk_max8(u[k]) : -INFINITY;
                tm = fmaxf(tm, cm[k]);   // a NaN chunk max (all NaN) loses
            }
            if (tm > b.v) {
                int kk = 0;
#pragma unroll
                for (int k = 7; k >= 0; --k) kk = (cm[k] == tm) ? k : kk;
                uint4 w = u[0];
#pragma unroll
                for (int k = 1; k < 8; ++k) w = (k == kk) ? u[k] : w;
                b.v = tm;
                b.i = 8 * (c + kk * kArgThreads) + first_equal8(w, tm);
            } else if (b.i == INT_MAX) {
                b.i = 8 * c;   // nothing above -inf yet: this batch's first element
            }
        }
        for (int i = c_hi * 8 + threadIdx.x; i < hi; i += kArgThreads) arg_take(b, __bfloat162float(x[i]), i);
    } else {
        for (int i = lo + threadIdx.x; i < hi; i += kArgThreads) arg_take(b, __bfloat162float(x[i]), i);
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ArgBest t{__shfl_xor_sync(0xffffffffu, b.v, o), __shfl_xor_sync(0xffffffffu, b.i, o)};
        arg_take(b, t.v, t.i);
    }
    __shared__ ArgBest s_best[kArgThreads / 32];
    if (threadIdx.x % 32 == 0) s_best[threadIdx.x / 32] = b;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kArgThreads / 32; ++w) arg_take(b, s_best[w].v, s_best[w].i);
        part_v[row * n_slices + s] = b.v;
        part_i[row * n_slices + s] = b.i;
    }
}

// One CTA (kTMax threads, thread i = node i) per sequence b.
__global__ void __launch_bounds__(kThreads)
accept_kernel(AcceptParams p) {
    __shared__ int s_jump[kTMax];
    __shared__ uint32_t s_anc[kTMax][kMaskWords];
    __shared__ int s_flag;
    __shared__ int s_amax[kTMax + 1];
    __shared__ uint32_t s_match[kMaskWords];
    __shared__ int s_best;
    const int b = blockIdx.x, i = threadIdx.x, T = p.T, W = (T + 31) / 32;
    // the mask needs only parent[]: built while the argmax grid runs
    const bool bad = build_tree_mask(p.parent + static_cast<size_t>(b) * T, T, s_jump, s_anc, &s_flag);
    if (i < kMaskWords) s_match[i] = 0u;
    if (i == 0) s_best = -1;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // argmax of row r of this sequence from its slices: warp w takes rows
    // w, w + 8, ..., four rows at a time, lane s reads slice s (n_slices <= 32),
    // so the partials of four rows are in flight at once
    {
        const int lane = i % 32, warp = i / 32;
        const size_t row0 = static_cast<size_t>(b) * (T + 1);
        for (int r0 = warp; r0 <= T; r0 += 4 * kWarps) {
            ArgBest c[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = r0 + u * kWarps;
                const bool live = r <= T && lane < p.n_slices;
                const size_t k = (row0 + r) * p.n_slices + lane;
                c[u].v = live ? p.part_v[k] : -INFINITY;
                c[u].i = live ? p.part_i[k] : INT_MAX;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float v = __shfl_xor_sync(0xffffffffu, c[u].v, o);
                    const int ix = __shfl_xor_sync(0xffffffffu, c[u].i, o);
                    arg_take(c[u], v, ix);
                }
                const int r = r0 + u * kWarps;
                if (lane == 0 && r <= T) s_amax[r] = c[u].i == INT_MAX ? 0 : c[u].i;
            }
        }
    }
    __syncthreads();
    if (i < T && !bad) {
        const int par = p.parent[static_cast<size_t>(b) * T + i];
        if (p.draft_tokens[static_cast<size_t>(b) * T + i] == s_amax[par < 0 ? 0 : par + 1])
            atomicOr(&s_match[i / 32], 1u << (i % 32));
    }
    __syncthreads();
    int depth = 0;
    if (i < T && !bad) {
        bool accepted = true;
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w)
            if (w < W) {
                depth += __popc(s_anc[i][w]);
                accepted = accepted && (s_anc[i][w] & ~s_match[w]) == 0u;
            }
        // deepest first, then the smallest id
        if (accepted) atomicMax(&s_best, (depth << 16) | (0xFFFF - i));
    }
    __syncthreads();
    const int best = s_best < 0 ? -1 : 0xFFFF - (s_best & 0xFFFF);
    const int len = best < 0 ? 0 : s_best >> 16;
    int32_t *path = p.path + static_cast<size_t>(b) * T;
    if (i < T) {
        if (i >= len) path[i] = -1;
        if (best >= 0 && (s_anc[best][i / 32] >> (i % 32) & 1u)) path[depth - 1] = i;
    }
    if (i == 0) {
        p.accept_len[b] = len;
        p.bonus[b] = s_amax[best < 0 ? 0 : best + 1];
        if (bad) raise_status(p.status, kStatusBadParent);
    }
}

cudaError_t launch_accept(const AcceptParams &p, cudaStream_t stream) {
    const int rows = p.B * (p.T + 1);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.stream = stream;
    cfg.gridDim = dim3(p.n_slices, rows);
    cfg.blockDim = dim3(kArgThreads);
    cudaError_t e = cudaLaunchKernelEx(&cfg, argmax_slices_kernel, p.logits, p.V, p.slice, p.part_v, p.part_i);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(p.B);
    cfg.blockDim = dim3(kThreads);
    return cudaLaunchKernelEx(&cfg, accept_kernel, p);
}

cudaError_t launch_tree_merge(const TreeMergeParams &p, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    if (p.mode == kTreeModeMask) {
        cfg.gridDim = dim3(1, 1, p.B);
    } else {
        const int M = (p.Hq / p.Hkv) * p.T;
        cfg.gridDim = dim3((M + kTreeRowsPerCta - 1) / kTreeRowsPerCta, p.Hkv, p.B);
    }
    if (p.mode == kTreeModeMerge || p.mode == kTreeModePrefixOnly) {
        // may start while the prefix kernel finishes; the merge waits for it
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, tree_merge_kernel, p);
}

}  // namespace hta
