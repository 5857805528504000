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
// Tensor memory (512 columns x 128 lanes):
//   S[0], S[1]  cols   0..255  fp32 scores of two tiles in flight; P (bf16
//                              pairs) is written back over them
//   O           cols 256..     fp32 output accumulator (D columns)
//   Q           after O        the Q tile as bf16 pairs (D/2 columns)
// Q sits in tensor memory so that Q K^T reads only K from shared memory:
// with both operands in shared memory a 128x128x16 MMA needs the SM's whole
// shared-memory bandwidth and the tensor pipe starves.
// Per tile j:  S[j%2] = Q K_j^T (A from tensor memory, B = K), then each
// softmax group reads its 64 score columns (one row per thread, no
// shuffles), the two groups exchange their row maxima through shared memory,
// write P, and O += P V_j (A = P from tensor memory, B = V, N-major).  O is
// rescaled only when the running max grew by more than 2^8 (a stale max is
// exact after the final normalisation; P stays <= 256).
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
    // barriers: q_full, q_tmem, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS],
    //           s_full[2], p_ready[2], o_ready, o_final, drain
    static constexpr int NUM_BARS = 2 + 4 * NS + 2 + 2 + 3;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;   // tmem base (4), abort flag (4)
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;    // slack to align the base to 1024
    // Once Q is in tensor memory its shared-memory tile is free: the row-max
    // exchange [parity][group][row] and the epilogue sums [group][2][row]
    // live there (first written after the first S tile, i.e. after every
    // warp has finished copying Q).
    static constexpr int OFF_RED = OFF_Q;
    static constexpr int OFF_SUMS = OFF_Q + 2 * 2 * 128 * 4;
    static constexpr int TMEM_COLS = 512;
    static constexpr int COL_S = 0;                         // S[b] at COL_S + 128*b
    static constexpr int COL_O = 256;
    static constexpr int COL_Q = COL_O + D;
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
    static_assert(COL_Q + D / 2 <= TMEM_COLS, "tensor memory budget");
    static_assert(OFF_SUMS + 2 * 2 * 128 * 4 <= Q_BYTES, "scratch inside the Q tile");
};

constexpr int kThreadsTc = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;

struct Bars {
    uint64_t *q_full, *q_tmem, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_ready,
             *o_ready, *o_final, *drain;
};

template <int NS>
__device__ __forceinline__ Bars carve_bars(uint64_t *base) {
    Bars b;
    b.q_full = base;
    b.q_tmem = base + 1;
    b.k_full = base + 2;
    b.k_empty = b.k_full + NS;
    b.v_full = b.k_empty + NS;
    b.v_empty = b.v_full + NS;
    b.s_full = b.v_empty + NS;      // [2]
    b.p_ready = b.s_full + 2;       // [2]
    b.o_ready = b.p_ready + 2;
    b.o_final = b.o_ready + 1;
    b.drain = b.o_final + 1;
    return b;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// packed pairs of fp32 (sm_100 f32x2 arithmetic)
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 unf2(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// A bounded wait whose outcome is the same on every lane of the warp, so
// that warp-collective instructions after it never see divergent lanes.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
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

    if (threadIdx.x == 0) {
        mbar_init(bars.q_full, 1);
        mbar_init(bars.q_tmem, 8);
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(bars.k_full + i, 1);
            mbar_init(bars.k_empty + i, 1);
            mbar_init(bars.v_full + i, 1);
            mbar_init(bars.v_empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bars.s_full + i, 1);
            mbar_init(bars.p_ready + i, 8);   // one arrive per softmax warp
        }
        mbar_init(bars.o_ready, 1);
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
        bool ok = warp_wait(bars.q_tmem, 0);
        tc_fence_after();
        for (int j = 0; ok && j <= n_tiles; ++j) {
            if (__any_sync(0xffffffffu, *s_abort != 0)) { ok = false; break; }
            if (j < n_tiles) {
                // S[j%2] = Q K_j^T : A = Q from tensor memory, B = K (K-major)
                const int st = j % C::NS;
                const uint32_t ph = (j / C::NS) & 1;
                const int sb = j & 1;
                if (!warp_wait(bars.k_full + st, ph)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t sk = smem_u32(smem + C::OFF_K + st * C::KV_BYTES);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
                        mma_ts(tmem + C::COL_S + sb * 128, tmem + C::COL_Q + kk * 8,
                               smem_desc_sw128(sk + off, 16, 1024), C::IDESC_QK, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bars.k_empty + st);
                    mma_commit(bars.s_full + sb);
                }
                __syncwarp();
            }
            if (j >= 1) {
                // O += P_{j-1} V_{j-1} : A = P from tensor memory, B = V (N-major)
                const int jj = j - 1;
                const int st = jj % C::NS;
                const uint32_t ph = (jj / C::NS) & 1;
                const int sb = jj & 1;
                if (!warp_wait(bars.v_full + st, ph)) { ok = false; break; }
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
                if (!warp_wait(bars.p_ready + sb, (jj >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t svu = smem_u32(sv);
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk) {
                        // P of keys 16kk..16kk+15: group kk/4 wrote it at its columns
                        const uint32_t a = tmem + C::COL_S + sb * 128 + (kk >> 2) * 64 + (kk & 3) * 8;
                        const uint64_t bdesc = smem_desc_sw128(svu + kk * 16 * 128, C::BOX_BYTES, 1024);
                        mma_ts(tmem + C::COL_O, a, bdesc, C::IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(bars.o_ready);
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
        const uint32_t t_o = tmem + lane_addr + C::COL_O + grp * (D / 2);
        float *red = reinterpret_cast<float *>(smem + C::OFF_RED);
        const float c2 = p.scale_log2;
        bool ok = true;

        // Q tile: shared memory (TMA, 128-byte swizzle) -> tensor memory.
        // Group g copies the g-th 64-column half of its row.
        if (!warp_wait(bars.q_full, 0)) { ok = false; abort_cta(); }
        if (ok && grp < C::HALVES) {
            const uint8_t *qrow = smem + C::OFF_Q + grp * C::BOX_BYTES + r * 128;
            uint32_t v[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 x = *reinterpret_cast<const uint4 *>(qrow + ((c ^ (r & 7)) << 4));
                v[4 * c + 0] = x.x;
                v[4 * c + 1] = x.y;
                v[4 * c + 2] = x.z;
                v[4 * c + 3] = x.w;
            }
            tmem_st32(tmem + lane_addr + C::COL_Q + grp * 32, v);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.q_tmem);

        float m_run = -INFINITY;      // running max of the scaled log2 scores (possibly stale)
        uint64_t l_exact = 0;         // pair of fp32 partial sums of 2^(x - m_run)
        uint64_t l_round = 0;         // the same over the bf16-rounded P that P*V uses
        for (int j = 0; j < n_tiles; ++j) {
            if (__any_sync(0xffffffffu, *s_abort != 0)) ok = false;
            const int sb = j & 1;
            if (ok && !warp_wait(bars.s_full + sb, (j >> 1) & 1)) { ok = false; abort_cta(); }
            tc_fence_after();
            const int n_valid = (j == n_tiles - 1) ? last_valid : C::BN;
            float s[64];
            float mloc = -INFINITY;
            if (ok && warp_active) {
                uint32_t ra[32], rb[32];
                tmem_ld32(t_s + sb * 128, ra);
                tmem_ld32(t_s + sb * 128 + 32, rb);
                tmem_wait_ld();
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
                float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
                for (int i = 4; i < 64; i += 8) {
                    m4[0] = max3(m4[0], s[i], s[i + 4]);
                    m4[1] = max3(m4[1], s[i + 1], s[i + 5]);
                    m4[2] = max3(m4[2], s[i + 2], s[i + 6]);
                    m4[3] = max3(m4[3], s[i + 3], s[i + 7]);
                }
                mloc = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
            }
            // row max over all 128 keys of the tile: exchange with the other group
            red[((j & 1) * 2 + grp) * 128 + r] = mloc;
            named_bar_sync(1, 256);
            const float mt = fmaxf(red[((j & 1) * 2 + 0) * 128 + r], red[((j & 1) * 2 + 1) * 128 + r]);
            if (ok && warp_active) {
                const float m_new = fmaxf(m_run, mt * c2);
                bool resc = false;
                float alpha = 1.f;
                if (m_new > m_run + 8.f) {
                    alpha = ex2(m_run - m_new);            // 0 on the first tile
                    l_exact = f2(unf2(l_exact).x * alpha, unf2(l_exact).y * alpha);
                    l_round = f2(unf2(l_round).x * alpha, unf2(l_round).y * alpha);
                    resc = j > 0;
                    m_run = m_new;
                }
                if (__any_sync(0xffffffffu, resc)) {
                    // O must hold P*V of tile j-1 before this group rescales its columns
                    if (!warp_wait(bars.o_ready, (j - 1) & 1)) { ok = false; abort_cta(); }
                    tc_fence_after();
                    const float a = resc ? alpha : 1.f;
#pragma unroll 1
                    for (int c = 0; c < D / 2; c += 32) {
                        uint32_t ro[32];
                        tmem_ld32(t_o + c, ro);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ro[i] = __float_as_uint(__uint_as_float(ro[i]) * a);
                        tmem_st32(t_o + c, ro);
                    }
                }
                const float mu = (m_run == -INFINITY) ? 0.f : m_run;
                const uint64_t cc = f2(c2, c2), nm = f2(-mu, -mu);
                uint32_t pk[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float2 x = unf2(fma2(f2(s[2 * k], s[2 * k + 1]), cc, nm));
                    const float p0 = ex2(x.x), p1 = ex2(x.y);
                    pk[k] = pack_bf16x2(p0, p1);
                    l_exact = add2(l_exact, f2(p0, p1));
                    l_round = add2(l_round, f2(bf16_lo(pk[k]), bf16_hi(pk[k])));
                }
                tmem_st32(t_s + sb * 128, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.p_ready + sb);
        }

        // ------------------------------------------------------ epilogue
        if (ok && !warp_wait(bars.o_final, 0)) { ok = false; abort_cta(); }
        tc_fence_after();
        float *sums = reinterpret_cast<float *>(smem + C::OFF_SUMS);   // [group][exact|round][row]
        const float2 le = unf2(l_exact), lr = unf2(l_round);
        sums[(grp * 2 + 0) * 128 + r] = le.x + le.y;
        sums[(grp * 2 + 1) * 128 + r] = lr.x + lr.y;
        named_bar_sync(1, 256);
        const float l_ex = sums[0 * 128 + r] + sums[2 * 128 + r];
        const float l_rd = sums[1 * 128 + r] + sums[3 * 128 + r];
        const bool failed = !ok || *s_abort;
        const int rr = row0 + r;
        if (warp_active) {
            const float inv = 1.f / l_rd;
            float *dst = p.o_part + ((grow0 + r) * p.S + split) * D + grp * (D / 2);
#pragma unroll 1
            for (int c = 0; c < D / 2; c += 32) {
                uint32_t x[32];
                tmem_ld32(t_o + c, x);
                tmem_wait_ld();
                if (rr < p.M) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 v;
                        v.x = __uint_as_float(x[i + 0]) * inv;
                        v.y = __uint_as_float(x[i + 1]) * inv;
                        v.z = __uint_as_float(x[i + 2]) * inv;
                        v.w = __uint_as_float(x[i + 3]) * inv;
                        *reinterpret_cast<float4 *>(dst + c + i) = v;
                    }
                }
            }
            if (grp == 0 && rr < p.M)
                p.lse_part[(grow0 + r) * p.S + split] = failed ? nan : (m_run + lg2(l_ex)) * kLn2;
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
