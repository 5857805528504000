// prefix_tc.cu -- split-KV prefix attention on sm_100a tensor cores.
//
// The prefix pass of Hybrid Tree Attention: every speculated tree token
// attends to the long shared prefix KV cache with no mask (LongSpec paper
// summary, "Summary", Hybrid Tree Attention bullet: "a Flash Attention pass
// over the prefix"; LongSpec README, "Introduction": fast prefix
// computation).  The KV range is cut into chunks (the split-KV of
// Flash-Decoding, cited by the same page) so that one call fills the GPU;
// each chunk yields a normalised partial O_c and its lse_c, merged later.
//
// CTA = one 128-row tile of the packed query group (rows r = g*T + t of the
// G query heads sharing KV head kvh) x one KV chunk, so the G*T rows share
// every K/V tile they read.  Warp roles (320 threads):
//   warps 0-3  softmax group 0: keys  0..63 of every 128-key tile
//   warps 4-7  softmax group 1: keys 64..127 of every 128-key tile
//   warp  8    TMA producer: Q once, then K and V tiles into NS-stage rings
//   warp  9    MMA issuer (one lane) and tensor-memory owner
// Tensor memory (512 columns x 128 lanes, fp32):
//   S[0], S[1]  cols   0..255  scores of two tiles in flight (double buffer);
//                              P (bf16 pairs) is written back over S
//   O[0], O[1]  cols 256..     one output accumulator per softmax group
// Per tile j:  S[j%2] = Q K_j^T (tcgen05.mma, A and B from shared memory),
// then each softmax group reads its 64 score columns (one row per thread,
// no shuffles), keeps its own running max / sum, writes P, and the MMA warp
// accumulates O[g] += P[g] V_j[g-th 64 keys] (A = P from tensor memory,
// B = V, N-major).  The two groups are two independent online softmaxes over
// interleaved halves of every tile; they are combined once, in the
// epilogue, by log-sum-exp rescaling.  A group rescales its O only when its
// running max grew by more than 2^8 (a stale max is exact after the final
// normalisation; P stays <= 256).
#include "hta_kernels.h"

namespace hta {

namespace {

template <int D>
struct TcCfg {
    static constexpr int BM = 128;
    static constexpr int BN = kKeyTile;                     // 128 keys per tile
    static constexpr int NS = (D == 128) ? 3 : 4;           // K and V ring depth
    static constexpr int HALVES = D / 64;                   // 64-column swizzle boxes
    static constexpr int BOX_BYTES = 128 * 64 * 2;          // one 128-row x 64-col box
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
    // barriers: q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS],
    //           s_full[2], p_ready[2][2], o_ready[2], o_final, drain
    static constexpr int NUM_BARS = 1 + 4 * NS + 2 + 4 + 2 + 1 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;   // tmem base (4), abort flag (4)
    // the epilogue's row statistics (m, l per group and row) reuse the Q
    // tile, which no MMA reads once the last P*V has completed
    static constexpr int OFF_STATS = OFF_Q;
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;    // slack to align the base to 1024
    static constexpr int TMEM_COLS = 512;
    static constexpr int COL_S = 0;                         // S[b] at COL_S + 128*b
    static constexpr int COL_O = 256;                       // O[g] at COL_O + D*g
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
};

constexpr int kThreadsTc = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;

struct Bars {
    uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_ready, *o_ready,
             *o_final, *drain;
};

template <int NS>
__device__ __forceinline__ Bars carve_bars(uint64_t *base) {
    Bars b;
    b.q_full = base;
    b.k_full = base + 1;
    b.k_empty = b.k_full + NS;
    b.v_full = b.k_empty + NS;
    b.v_empty = b.v_full + NS;
    b.s_full = b.v_empty + NS;      // [2]
    b.p_ready = b.s_full + 2;       // [2 buffers][2 groups]
    b.o_ready = b.p_ready + 4;      // [2 groups]
    b.o_final = b.o_ready + 2;
    b.drain = b.o_final + 1;
    return b;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreadsTc, 1)
prefix_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const PrefixParams p) {
    using C = TcCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = blockIdx.x, split = blockIdx.y, bk = blockIdx.z;
    const int b = bk / p.Hkv;
    const int row0 = mt * C::BM;
    const size_t grow0 = static_cast<size_t>(bk) * p.M + row0;
    const float nan = __int_as_float(0x7fc00000);
    const int L = p.prefix_len[b];
    if (L < 0 || L > p.L_cap) {
        if (threadIdx.x < C::BM && row0 + static_cast<int>(threadIdx.x) < p.M)
            p.lse_part[(grow0 + threadIdx.x) * p.S + split] = nan;
        if (threadIdx.x == 0) raise_status(p.status, kStatusPrefixLenRange);
        return;
    }
    const int key_begin = split * p.chunk_tiles * C::BN;
    const int key_end = min(L, key_begin + p.chunk_tiles * C::BN);
    const int n_tiles = key_end > key_begin ? (key_end - key_begin + C::BN - 1) / C::BN : 0;
    if (n_tiles == 0) {   // chunk past the end of this sequence: an empty partial
        if (threadIdx.x < C::BM && row0 + static_cast<int>(threadIdx.x) < p.M)
            p.lse_part[(grow0 + threadIdx.x) * p.S + split] = -INFINITY;
        return;
    }
    const int last_valid = key_end - (key_begin + (n_tiles - 1) * C::BN);   // 1..128

    Bars bars = carve_bars<C::NS>(reinterpret_cast<uint64_t *>(smem + C::OFF_BAR));
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    float *s_stat = reinterpret_cast<float *>(smem + C::OFF_STATS);   // [group][m|l][128]

    if (threadIdx.x == 0) {
        mbar_init(bars.q_full, 1);
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(bars.k_full + i, 1);
            mbar_init(bars.k_empty + i, 1);
            mbar_init(bars.v_full + i, 1);
            mbar_init(bars.v_empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) mbar_init(bars.s_full + i, 1);
        for (int i = 0; i < 4; ++i) mbar_init(bars.p_ready + i, 128);
        for (int i = 0; i < 2; ++i) mbar_init(bars.o_ready + i, 1);
        mbar_init(bars.o_final, 1);
        mbar_init(bars.drain, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(s_tmem, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    auto abort_cta = [&]() {
        *s_abort = 1;
        raise_status(p.status, kStatusPipelineTimeout);
    };

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            uint8_t *sq = smem + C::OFF_Q;
            mbar_arrive_expect_tx(bars.q_full, C::Q_BYTES);
#pragma unroll
            for (int h = 0; h < C::HALVES; ++h)
                tma_load_2d(sq + h * C::BOX_BYTES, &tm_q, bars.q_full, h * 64, static_cast<int>(grow0));
            const int kv_row0 = bk * p.L_cap + key_begin;
            int k_issued = 0, v_issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int st = j % C::NS;
                const uint32_t ph = (j / C::NS) & 1;
                if (*s_abort) break;
                if (!mbar_wait(bars.k_empty + st, ph ^ 1)) { abort_cta(); break; }
                uint8_t *sk = smem + C::OFF_K + st * C::KV_BYTES;
                mbar_arrive_expect_tx(bars.k_full + st, C::KV_BYTES);
#pragma unroll
                for (int h = 0; h < C::HALVES; ++h)
                    tma_load_2d(sk + h * C::BOX_BYTES, &tm_k, bars.k_full + st, h * 64, kv_row0 + j * C::BN);
                k_issued = j + 1;
                if (!mbar_wait(bars.v_empty + st, ph ^ 1)) { abort_cta(); break; }
                uint8_t *sv = smem + C::OFF_V + st * C::KV_BYTES;
                mbar_arrive_expect_tx(bars.v_full + st, C::KV_BYTES);
#pragma unroll
                for (int h = 0; h < C::HALVES; ++h)
                    tma_load_2d(sv + h * C::BOX_BYTES, &tm_v, bars.v_full + st, h * 64, kv_row0 + j * C::BN);
                v_issued = j + 1;
            }
            if (*s_abort) {
                // let the copies in flight land before the CTA releases its smem
                for (int j = max(0, k_issued - C::NS); j < k_issued; ++j)
                    mbar_wait(bars.k_full + j % C::NS, (j / C::NS) & 1);
                for (int j = max(0, v_issued - C::NS); j < v_issued; ++j)
                    mbar_wait(bars.v_full + j % C::NS, (j / C::NS) & 1);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA
        bool ok = mbar_wait(bars.q_full, 0);
        tc_fence_after();
        const uint32_t sq = smem_u32(smem + C::OFF_Q);
        for (int j = 0; ok && j <= n_tiles; ++j) {
            if (*s_abort) { ok = false; break; }
            if (j < n_tiles) {
                const int st = j % C::NS;
                const uint32_t ph = (j / C::NS) & 1;
                const int sb = j & 1;
                if (!mbar_wait(bars.k_full + st, ph)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t sk = smem_u32(smem + C::OFF_K + st * C::KV_BYTES);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
                        mma_ss(tmem + C::COL_S + sb * 128, smem_desc_sw128(sq + off, 16, 1024),
                               smem_desc_sw128(sk + off, 16, 1024), C::IDESC_QK, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bars.k_empty + st);
                    mma_commit(bars.s_full + sb);
                }
                __syncwarp();
            }
            if (j >= 1) {
                const int jj = j - 1;
                const int st = jj % C::NS;
                const uint32_t ph = (jj / C::NS) & 1;
                const int sb = jj & 1;
                if (!mbar_wait(bars.v_full + st, ph)) { ok = false; break; }
                uint8_t *sv = smem + C::OFF_V + st * C::KV_BYTES;
                if (jj == n_tiles - 1 && last_valid < C::BN) {
                    // keys past L_b may hold anything (even NaN): zero their V
                    // rows so that P = 0 really contributes nothing
                    const int per_row = C::HALVES * 8;   // 16-byte chunks per key row
                    for (int idx = lane; idx < (C::BN - last_valid) * per_row; idx += 32) {
                        const int r = last_valid + idx / per_row;
                        const int h = (idx % per_row) / 8, c = idx % 8;
                        *reinterpret_cast<uint4 *>(sv + h * C::BOX_BYTES + r * 128 + c * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                const uint32_t svu = smem_u32(sv);
                for (int g = 0; g < 2; ++g) {
                    if (!mbar_wait(bars.p_ready + sb * 2 + g, (jj >> 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    if (lane == 0) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const int key0 = g * 64 + kk * 16;
                            const uint64_t bdesc = smem_desc_sw128(svu + key0 * 128, C::BOX_BYTES, 1024);
                            mma_ts(tmem + C::COL_O + g * D, tmem + C::COL_S + sb * 128 + g * 64 + kk * 8,
                                   bdesc, C::IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(bars.o_ready + g);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) {
                    mma_commit(bars.v_empty + st);
                    if (jj == n_tiles - 1) mma_commit(bars.o_final);
                }
                __syncwarp();
            }
        }
        if (!ok) abort_cta();
        // every MMA this warp issued must be complete before TMEM is freed
        if (lane == 0) {
            mma_commit(bars.drain);
            mbar_wait(bars.drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- softmax
        const int grp = warp >> 2, wq = warp & 3;
        const int r = wq * 32 + lane;                       // row of the tile = TMEM lane
        const bool warp_active = row0 + wq * 32 < p.M;      // any real row in this warp
        const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t t_s = tmem + lane_addr + C::COL_S + grp * 64;
        const uint32_t t_o = tmem + lane_addr + C::COL_O + grp * D;
        const float c2 = p.scale_log2;
        float m_run = -INFINITY;   // running max of the scaled log2 scores (possibly stale)
        float l_run = 0.f;         // running sum of 2^(score - m_run)
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            if (*s_abort) { ok = false; break; }
            const int sb = j & 1;
            if (!mbar_wait(bars.s_full + sb, (j >> 1) & 1)) { ok = false; abort_cta(); break; }
            tc_fence_after();
            const int n_valid = (j == n_tiles - 1) ? last_valid : C::BN;
            if (warp_active) {
                uint32_t ra[32], rb[32];
                tmem_ld32(t_s + sb * 128, ra);
                tmem_ld32(t_s + sb * 128 + 32, rb);
                tmem_wait_ld();
                float s[64];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    s[i] = __uint_as_float(ra[i]);
                    s[32 + i] = __uint_as_float(rb[i]);
                }
                if (n_valid < C::BN) {
                    const int lim = n_valid - grp * 64;
#pragma unroll
                    for (int i = 0; i < 64; ++i) s[i] = (i < lim) ? s[i] : -INFINITY;
                }
                float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
                for (int i = 4; i < 64; i += 4) {
                    mx4[0] = fmaxf(mx4[0], s[i]);
                    mx4[1] = fmaxf(mx4[1], s[i + 1]);
                    mx4[2] = fmaxf(mx4[2], s[i + 2]);
                    mx4[3] = fmaxf(mx4[3], s[i + 3]);
                }
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                const float m_new = fmaxf(m_run, mx * c2);
                bool resc = false;
                float alpha = 1.f;
                if (m_new > m_run + 8.f) {
                    alpha = ex2(m_run - m_new);            // 0 on the first tile
                    l_run *= alpha;
                    resc = j > 0;
                    m_run = m_new;
                }
                if (__any_sync(0xffffffffu, resc)) {
                    // O of this group must hold P*V of tile j-1 before it is rescaled
                    if (!mbar_wait(bars.o_ready + grp, (j - 1) & 1)) { ok = false; abort_cta(); }
                    tc_fence_after();
                    const float a = resc ? alpha : 1.f;
#pragma unroll 1
                    for (int c = 0; c < D; c += 32) {
                        uint32_t ro[32];
                        tmem_ld32(t_o + c, ro);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ro[i] = __float_as_uint(__uint_as_float(ro[i]) * a);
                        tmem_st32(t_o + c, ro);
                    }
                }
                const float mu = (m_run == -INFINITY) ? 0.f : m_run;
                uint32_t pk[32];
                float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float p0 = ex2(fmaf(s[2 * k], c2, -mu));
                    const float p1 = ex2(fmaf(s[2 * k + 1], c2, -mu));
                    ls0 += p0;
                    ls1 += p1;
                    pk[k] = pack_bf16x2(p0, p1);
                }
                l_run += ls0 + ls1;
                tmem_st32(t_s + sb * 128, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bars.p_ready + sb * 2 + grp);
            if (!ok) break;
        }

        // ------------------------------------------------------ epilogue
        if (ok && !mbar_wait(bars.o_final, 0)) { ok = false; abort_cta(); }
        tc_fence_after();
        named_bar_sync(1, 256);   // every MMA is done: the Q tile may be reused
        s_stat[(grp * 2 + 0) * 128 + r] = m_run;
        s_stat[(grp * 2 + 1) * 128 + r] = l_run;
        named_bar_sync(1, 256);
        const float m0 = s_stat[0 * 128 + r], l0 = s_stat[1 * 128 + r];
        const float m1 = s_stat[2 * 128 + r], l1 = s_stat[3 * 128 + r];
        const float mx = fmaxf(m0, m1);
        const float a0 = ex2(m0 - mx), a1 = ex2(m1 - mx);
        const float lt = l0 * a0 + l1 * a1;
        const float f0 = a0 / lt, f1 = a1 / lt;
        const bool failed = !ok || *s_abort;
        const int rr = row0 + r;
        if (warp_active) {
            float *dst = p.o_part + ((grow0 + r) * p.S + split) * D;
#pragma unroll 1
            for (int c = grp * (D / 2); c < (grp + 1) * (D / 2); c += 32) {
                uint32_t x0[32], x1[32];
                tmem_ld32(tmem + lane_addr + C::COL_O + c, x0);
                tmem_ld32(tmem + lane_addr + C::COL_O + D + c, x1);
                tmem_wait_ld();
                if (rr < p.M) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 v;
                        v.x = f0 * __uint_as_float(x0[i + 0]) + f1 * __uint_as_float(x1[i + 0]);
                        v.y = f0 * __uint_as_float(x0[i + 1]) + f1 * __uint_as_float(x1[i + 1]);
                        v.z = f0 * __uint_as_float(x0[i + 2]) + f1 * __uint_as_float(x1[i + 2]);
                        v.w = f0 * __uint_as_float(x0[i + 3]) + f1 * __uint_as_float(x1[i + 3]);
                        *reinterpret_cast<float4 *>(dst + c + i) = v;
                    }
                }
            }
            if (grp == 0 && rr < p.M)
                p.lse_part[(grow0 + r) * p.S + split] = failed ? nan : (mx + lg2(lt)) * kLn2;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D>
cudaError_t launch_tc(const PrefixParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                      const CUtensorMap &tm_v, cudaStream_t stream) {
    using C = TcCfg<D>;
    static_assert(C::SMEM_ALLOC <= 232448, "shared memory budget");
    constexpr int kMaxDev = 64;
    static bool attr_set[kMaxDev] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev || !attr_set[dev]) {
        e = cudaFuncSetAttribute(prefix_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_ALLOC);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < kMaxDev) attr_set[dev] = true;
    }
    dim3 grid(p.m_tiles, p.S, p.B * p.Hkv);
    prefix_tc_kernel<D><<<grid, kThreadsTc, C::SMEM_ALLOC, stream>>>(tm_q, tm_k, tm_v, p);
    return cudaGetLastError();
}

cudaError_t launch_prefix_tc(const PrefixParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                             const CUtensorMap &tm_v, cudaStream_t stream) {
    if (p.D == 128) return launch_tc<128>(p, tm_q, tm_k, tm_v, stream);
    return launch_tc<64>(p, tm_q, tm_k, tm_v, stream);
}

}  // namespace hta
