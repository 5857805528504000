// prefix_simt.cu -- plain CUDA-core split-KV prefix attention (no tensor
// cores, no TMA).  Same partials as the tcgen05 kernel; kept as an
// independent GPU cross-check of it, selected with
// LONGSPEC_HTA_PREFIX_SIMT.  The prefix pass itself is the unmasked
// "Flash Attention pass over the prefix" of the LongSpec paper summary
// ("Summary", Hybrid Tree Attention bullet), split over KV chunks as in
// Flash-Decoding (cited by the same page).
//
// One CTA = 8 warps = 8 packed rows of one (b, KV head) over one KV chunk.
// Keys are staged 32 at a time in shared memory; lane j scores key j, the
// warp keeps an online softmax (max, sum) and each lane accumulates D/32
// output columns.
#include "hta_kernels.h"

namespace hta {

namespace {

constexpr int kRows = 8;
constexpr int kSub = 32;

template <int D>
__global__ void __launch_bounds__(kRows * 32)
prefix_simt_kernel(PrefixParams p) {
    constexpr int DPL = D / 32;
    constexpr int RW = D / 2 + 1;                 // padded row stride in 32-bit words
    __shared__ uint32_t s_k[kSub * RW];
    __shared__ uint32_t s_v[kSub * RW];
    __shared__ float s_q[kRows][D];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int split = blockIdx.x, bk = blockIdx.z;
    const int b = bk / p.Hkv;
    const int rr = blockIdx.y * kRows + warp;
    const bool active = rr < p.M;
    const size_t row = static_cast<size_t>(bk) * p.M + rr;
    const int L = p.prefix_len[b];
    if (L < 0 || L > p.L_cap) {
        if (active && lane == 0) p.lse_part[row * p.S + split] = __int_as_float(0x7fc00000);
        if (threadIdx.x == 0) raise_status(p.status, kStatusPrefixLenRange);
        return;
    }
    const int k0 = split * p.chunk_tiles * kKeyTile;
    const int k1 = min(L, k0 + p.chunk_tiles * kKeyTile);

    for (int d = lane; d < D; d += 32)
        s_q[warp][d] = active ? __bfloat162float(p.q[row * D + d]) * p.scale_log2 : 0.f;

    float m = -INFINITY, l = 0.f, acc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
    const size_t kv_row0 = static_cast<size_t>(bk) * p.L_cap;
    const uint32_t *kg = reinterpret_cast<const uint32_t *>(p.k_prefix);
    const uint32_t *vg = reinterpret_cast<const uint32_t *>(p.v_prefix);

    for (int base = k0; base < k1; base += kSub) {
        const int n = min(kSub, k1 - base);
        __syncthreads();
        for (int idx = threadIdx.x; idx < kSub * (D / 2); idx += blockDim.x) {
            const int j = idx / (D / 2), c = idx % (D / 2);
            const bool ok = j < n;
            s_k[j * RW + c] = ok ? kg[(kv_row0 + base + j) * (D / 2) + c] : 0u;
            s_v[j * RW + c] = ok ? vg[(kv_row0 + base + j) * (D / 2) + c] : 0u;
        }
        __syncthreads();
        float dot = 0.f;
#pragma unroll 8
        for (int c = 0; c < D / 2; ++c) {
            const uint32_t kw = s_k[lane * RW + c];
            dot = fmaf(s_q[warp][2 * c], bf16_lo(kw), dot);
            dot = fmaf(s_q[warp][2 * c + 1], bf16_hi(kw), dot);
        }
        const float x = lane < n ? dot : -INFINITY;
        float mx = x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_new = fmaxf(m, mx);
        const float a = ex2(m - m_new);
        const float pj = ex2(x - m_new);
        float ps = pj;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        l = l * a + ps;
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[i] *= a;
        for (int j = 0; j < n; ++j) {
            const float pb = __shfl_sync(0xffffffffu, pj, j);
#pragma unroll
            for (int i = 0; i < DPL; i += 2) {
                const uint32_t vw = s_v[j * RW + (lane * DPL + i) / 2];
                acc[i] = fmaf(pb, bf16_lo(vw), acc[i]);
                acc[i + 1] = fmaf(pb, bf16_hi(vw), acc[i + 1]);
            }
        }
        m = m_new;
    }
    if (!active) return;
    float *o = p.o_part + (row * p.S + split) * D + lane * DPL;
    if (k1 <= k0) {
        if (lane == 0) p.lse_part[row * p.S + split] = -INFINITY;
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[i] = 0.f;
        return;
    }
    const float inv = 1.f / l;
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[i] = acc[i] * inv;
    if (lane == 0) p.lse_part[row * p.S + split] = (m + lg2(l)) * kLn2;
}

}  // namespace

cudaError_t launch_prefix_simt(const PrefixParams &p, cudaStream_t stream) {
    dim3 grid(p.S, (p.M + kRows - 1) / kRows, p.B * p.Hkv);
    if (p.D == 128) prefix_simt_kernel<128><<<grid, kRows * 32, 0, stream>>>(p);
    else prefix_simt_kernel<64><<<grid, kRows * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace hta
