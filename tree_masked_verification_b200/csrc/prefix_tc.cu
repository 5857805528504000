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
// every K/V tile they read.  Warp roles (384 threads, three warpgroups):
//   warp  0    TMA producer of Q and the K ring
//   warp  1    MMA issuer (one lane) and tensor-memory owner
//   warp  2    TMA producer of the V ring
//   warp  3    idle (completes the first warpgroup)
//   warps 4-7  softmax group 0: the even key tiles of the chunk
//   warps 8-11 softmax group 1: the odd key tiles
// Warp w reaches tensor-memory lanes 32(w%4)..32(w%4)+31 and runs on
// sub-partition w%4.  The MMA issuer shares its sub-partition with two
// softmax warps; it has the lower warp index of the three.
// The first warpgroup hands registers to the softmax warpgroups
// (setmaxnreg): 2 x 128 x 224 + 128 x 56 = 384 x 168, the launch budget.
// Each group runs its own online softmax (running max m_g, sums l_g) into
// its own accumulator O_g; the epilogue merges the two exactly, as the lse
// merge of two KV ranges.  The groups therefore never wait for each other,
// and the two warps that share an SM sub-partition (w and w+4) work on
// different tiles, so one of them keeps the exp2 unit busy while the
// other loads scores and takes its row max.
// Tensor memory (512 columns x 128 lanes):
//   S[g]   cols 128g..128g+127  fp32 scores of group g's current tile; P
//                               (bf16 pairs) is written back over them
//   O[g]   cols 256+gD..        fp32 accumulator of group g (D columns)
// Per tile j (group g = j%2):  S[g] = Q K_j^T (both operands in shared
// memory); every thread of group g reads the 128 scores of its row (one row
// per thread, no shuffles), takes the row max and writes P over the first
// 64 columns of S[g].  Then O[g] += P V_j (A = P from tensor memory, B = V,
// N-major).  The running max moves only when it grew by more than 2^8 (a
// stale max is exact after the final normalisation; P stays <= 256); O[g]
// is rescaled then.
#include "hta_kernels.h"

namespace hta {

namespace {

template <int D>
struct TcCfg {
    static constexpr int BM = 128;
    static constexpr int BN = kKeyTile;                     // 128 keys per tile
    static constexpr int NS = (D == 128) ? HTA_KV_STAGES_D128 : 4;   // K and V ring depth
    static constexpr int HALVES = D / 64;                   // 64-column swizzle boxes
    static constexpr int BOX_BYTES = 128 * 64 * 2;          // one 128-row x 64-col box
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
    // barriers: q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS],
    //           v_tail, s_full[2], p_ready[2], o_final, drain
    static constexpr int NUM_BARS = 1 + 4 * NS + 1 + 2 + 2 + 2;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;   // tmem base (4), abort flag (4)
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;    // slack to align the base to 1024
    // After the last MMA the K and V rings are free: the epilogue exchanges
    // the groups' per-row statistics [group][m|l_exact|l_round][row] in the
    // first K stage and stages the output rows [row][D] fp32 in the V ring.
    static constexpr int OFF_XCH = OFF_K;
    static constexpr int OFF_STAGE = OFF_V;
    static constexpr int TMEM_COLS = 512;
    static constexpr int COL_S = 0;                         // S[g] at COL_S + 128*g
    static constexpr int COL_O = 256;                       // O[g] at COL_O + D*g
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
    static_assert(COL_O + 2 * D <= TMEM_COLS, "tensor memory budget");
    static_assert(2 * 3 * 128 * 4 <= KV_BYTES, "statistics exchange inside one K stage");
    static_assert(BM * D * 4 <= NS * KV_BYTES, "output staging inside the V ring");
};

constexpr int kThreadsTc = 384;
constexpr int kRegsSoftmax = 224;   // per thread, softmax warpgroups
constexpr int kRegsOther = 56;      // per thread, producer / MMA warpgroup
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreadsTc * 168,
              "register split must fit the launch allocation");
constexpr int kProducerKWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kProducerVWarp = 2;
constexpr int kFirstSoftmaxWarp = 4;

struct Bars {
    uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *v_tail, *s_full, *p_ready,
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
    b.v_tail = b.v_empty + NS;
    b.s_full = b.v_tail + 1;        // [2], one per group
    b.p_ready = b.s_full + 2;       // [2]
    b.o_final = b.p_ready + 2;
    b.drain = b.o_final + 1;
    return b;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// bar.sync over `nthreads` threads that also returns, on every one of them,
// whether any of them passed `pred` true
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %3, 0;\n\t"
        "bar.red.or.pred q, %1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r) : "r"(id), "r"(nthreads), "r"(pred ? 1u : 0u) : "memory");
    return r != 0;
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

template <int N>
__device__ __forceinline__ void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }

// 2^x for a pair on the FMA pipe, to take part of the load off the exp2
// unit: n = round(x) by the 1.5 * 2^23 addition, f = x - n in [-1/2, 1/2],
// 2^f by the cubic fitted in fit_exp2_poly.py (relative error 7.5e-5, far
// below bf16's 2^-9), then n added to the exponent field.  x is clamped to
// >= -125 so that the result stays a normal number (2^-125 is 0 for every
// sum here); x <= 2^8 always holds (lazy max).
__device__ __forceinline__ float2 exp2_poly2(uint64_t x2) {
    constexpr float kRound = 12582912.0f;    // 1.5 * 2^23
    float2 v = unf2(x2);
    v.x = fmaxf(v.x, -125.f);
    v.y = fmaxf(v.y, -125.f);
    const uint64_t xc = f2(v.x, v.y);
    const uint64_t t = add2(xc, f2(kRound, kRound));            // n in the low mantissa bits
    const uint64_t n = add2(t, f2(-kRound, -kRound));            // n as a float, exact
    const uint64_t fr = fma2(n, f2(-1.f, -1.f), xc);             // f = x - n, exact
    uint64_t q = fma2(fr, f2(0.05517132207751274f, 0.05517132207751274f),
                      f2(0.24261054396629333f, 0.24261054396629333f));
    q = fma2(fr, q, f2(0.6932609677314758f, 0.6932609677314758f));
    q = fma2(fr, q, f2(0.9999281167984009f, 0.9999281167984009f));
    const float2 qq = unf2(q), tt = unf2(t);
    float2 o;
    o.x = __int_as_float(__float_as_int(qq.x) + (__float_as_int(tt.x) << 23));
    o.y = __int_as_float(__float_as_int(qq.y) + (__float_as_int(tt.y) << 23));
    return o;
}

// L2 eviction policies (createpolicy) and the hinted TMA load / store
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void tma_load_2d_hint(void *smem_dst, const CUtensorMap *map, uint64_t *bar,
                                                 int x, int y, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)),
          "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(pol)
        : "memory");
}
__device__ __forceinline__ void st_v4_hint(float *dst, float4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;"
                 ::"l"(dst), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_f32_hint(float *dst, float v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(dst), "f"(v), "l"(pol) : "memory");
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

}  // namespace

template <int D, bool PAGED, bool WINDOW>
__global__ void __launch_bounds__(kThreadsTc, 1)
prefix_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const PrefixParams p) {
    using C = TcCfg<D>;
    // Launched with programmatic stream serialisation: the CTA may be
    // resident before the previous kernel on the stream has finished, so it
    // waits for that grid (and its memory) before touching any input.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = blockIdx.x, split = blockIdx.y, bk = blockIdx.z;
    const int b = bk / p.Hkv;
    const int row0 = mt * C::BM;
    const size_t grow0 = static_cast<size_t>(bk) * p.M + row0;
    const float nan = __int_as_float(0x7fc00000);
    const int L = p.prefix_len[b];
    if (L < 0 || (!WINDOW && L > p.L_cap)) {
        if (threadIdx.x < C::BM && row0 + static_cast<int>(threadIdx.x) < p.M)
            p.lse_part[(grow0 + threadIdx.x) * p.S + split] = nan;
        if (threadIdx.x == 0) raise_status(p.status, kStatusPrefixLenRange);
        return;
    }
    // (sliding window: the chunks start at the tile holding L_b - W)
    const int key_begin = (WINDOW ? max(0, L - p.window) / C::BN * C::BN : 0) + split * p.chunk_tiles * C::BN;
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
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(bars.k_full + i, 1);
            mbar_init(bars.k_empty + i, 1);
            mbar_init(bars.v_full + i, 1);
            mbar_init(bars.v_empty + i, 1);
        }
        mbar_init(bars.v_tail, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bars.s_full + i, 1);
            mbar_init(bars.p_ready + i, 4);   // one arrive per warp of the group
        }
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
    // the tree pass may launch now: it only waits for this grid before merging
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    auto abort_cta = [&]() {
        *s_abort = 1;
        raise_status(p.status, kStatusPipelineTimeout);
    };
    const int kv_row0 = bk * p.L_cap + key_begin;
    // K/V read by one row tile only (G*T <= 128): each line is used once,
    // so it is marked first to leave L2, which keeps the split partials
    // (marked last) there until the merge reads them
    const bool stream_once = p.m_tiles == 1;
    // Producer of a K or V ring from a paged cache, run by the whole warp.
    // A 128-key tile is read with one block_size-row box per block and
    // 64-column half, each landing at the block's rows of the swizzled stage
    // (block_size * 128 bytes is a multiple of the 1024-byte swizzle period,
    // so the layout is that of one tall box).  Per tile, lane 0 waits for the
    // stage and posts the byte count; then lane i < 128/block_size issues the
    // boxes of block i, whose id it read from the table one tile earlier.
    // Blocks past L_b are read from the sequence's last block (their keys
    // are masked); an id outside [0, num_blocks) is read as block 0 and
    // flagged.  Returns the number of tiles issued.
    auto paged_ring = [&](uint8_t *ring, const CUtensorMap *map, uint64_t *full, uint64_t *empty) {
        const int bs = p.block_size, nb = kKeyTile / bs, kvh = bk % p.Hkv;
        const int32_t *row = p.block_table + static_cast<size_t>(b) * p.max_blocks;
        const int last = (L - 1) / bs;          // L >= 1: n_tiles > 0 here
        auto fetch = [&](int key0) { return lane < nb ? row[min(key0 / bs + lane, last)] : 0; };
        int id = fetch(key_begin);
        int issued = 0;
        for (int j = 0; j < n_tiles; ++j) {
            const int st = j % C::NS;
            int go = 0;                          // 1: proceed, 0: aborted, 2: wait ran out
            if (lane == 0) {
                go = *s_abort ? 0 : mbar_wait(empty + st, ((j / C::NS) & 1) ^ 1) ? 1 : 2;
                if (go == 1) mbar_arrive_expect_tx(full + st, C::KV_BYTES);
                if (go == 2) abort_cta();
            }
            go = __shfl_sync(0xffffffffu, go, 0);
            if (go != 1) break;
            if (lane < nb) {
                int n = id;
                if (n < 0 || n >= p.num_blocks) {
                    raise_status(p.status, kStatusBadBlock);
                    n = 0;
                }
                const int y = (n * p.Hkv + kvh) * bs;
                uint8_t *stage = ring + st * C::KV_BYTES + lane * bs * 128;
#pragma unroll
                for (int h = 0; h < C::HALVES; ++h) tma_load_2d(stage + h * C::BOX_BYTES, map, full + st, h * 64, y);
            }
            id = fetch(key_begin + (j + 1) * C::BN);   // the next tile's block
            issued = j + 1;
        }
        __syncwarp();
        return issued;
    };
    // Producer of a K or V ring from the sliding-window ring cache (one
    // thread): tile j holds context positions key_begin + j*128 + [0, 128),
    // which sit at slots (key_begin + j*128) mod W + [0, 128) of this KV
    // head's W-slot ring (W a multiple of 128, so a tile never wraps).
    auto window_ring = [&](uint8_t *ring, const CUtensorMap *map, uint64_t *full, uint64_t *empty) {
        int issued = 0;
        for (int j = 0; j < n_tiles; ++j) {
            const int st = j % C::NS;
            if (*s_abort) break;
            if (!mbar_wait(empty + st, ((j / C::NS) & 1) ^ 1)) { abort_cta(); break; }
            uint8_t *stage = ring + st * C::KV_BYTES;
            mbar_arrive_expect_tx(full + st, C::KV_BYTES);
            const int y = bk * p.window + (key_begin + j * C::BN) % p.window;
#pragma unroll
            for (int h = 0; h < C::HALVES; ++h) tma_load_2d(stage + h * C::BOX_BYTES, map, full + st, h * 64, y);
            issued = j + 1;
        }
        return issued;
    };
    if (warp == kProducerKWarp) {
        // -------------------------------------------------------- TMA: Q, K
        regs_dec<kRegsOther>();
        const uint64_t kv_pol = l2_policy_evict_first();
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            uint8_t *sq = smem + C::OFF_Q;
            mbar_arrive_expect_tx(bars.q_full, C::Q_BYTES);
#pragma unroll
            for (int h = 0; h < C::HALVES; ++h)
                tma_load_2d(sq + h * C::BOX_BYTES, &tm_q, bars.q_full, h * 64, static_cast<int>(grow0));
        }
        if constexpr (PAGED) {
            const int issued = paged_ring(smem + C::OFF_K, &tm_k, bars.k_full, bars.k_empty);
            if (lane == 0 && *s_abort) {
                mbar_wait(bars.q_full, 0);
                for (int j = max(0, issued - C::NS); j < issued; ++j)
                    mbar_wait(bars.k_full + j % C::NS, (j / C::NS) & 1);
            }
        } else if constexpr (WINDOW) {
            if (lane == 0) {
                const int issued = window_ring(smem + C::OFF_K, &tm_k, bars.k_full, bars.k_empty);
                if (*s_abort) {
                    mbar_wait(bars.q_full, 0);
                    for (int j = max(0, issued - C::NS); j < issued; ++j)
                        mbar_wait(bars.k_full + j % C::NS, (j / C::NS) & 1);
                }
            }
        } else if (lane == 0) {
            int issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int st = j % C::NS;
                if (*s_abort) break;
                if (!mbar_wait(bars.k_empty + st, ((j / C::NS) & 1) ^ 1)) { abort_cta(); break; }
                uint8_t *sk = smem + C::OFF_K + st * C::KV_BYTES;
                mbar_arrive_expect_tx(bars.k_full + st, C::KV_BYTES);
#pragma unroll
                for (int h = 0; h < C::HALVES; ++h) {
                    if (stream_once)
                        tma_load_2d_hint(sk + h * C::BOX_BYTES, &tm_k, bars.k_full + st, h * 64, kv_row0 + j * C::BN, kv_pol);
                    else
                        tma_load_2d(sk + h * C::BOX_BYTES, &tm_k, bars.k_full + st, h * 64, kv_row0 + j * C::BN);
                }
                issued = j + 1;
            }
            if (*s_abort) {
                // let the copies in flight land before the CTA releases its smem
                mbar_wait(bars.q_full, 0);
                for (int j = max(0, issued - C::NS); j < issued; ++j)
                    mbar_wait(bars.k_full + j % C::NS, (j / C::NS) & 1);
            }
        }
        __syncwarp();
    } else if (warp == kProducerVWarp) {
        // ----------------------------------------------------------- TMA: V
        regs_dec<kRegsOther>();
        const uint64_t kv_pol = l2_policy_evict_first();
        if (lane == 0) tma_prefetch_desc(&tm_v);
        if constexpr (PAGED) {
            const int issued = paged_ring(smem + C::OFF_V, &tm_v, bars.v_full, bars.v_empty);
            if (lane == 0 && *s_abort) {
                for (int j = max(0, issued - C::NS); j < issued; ++j)
                    mbar_wait(bars.v_full + j % C::NS, (j / C::NS) & 1);
            }
        } else if constexpr (WINDOW) {
            if (lane == 0) {
                const int issued = window_ring(smem + C::OFF_V, &tm_v, bars.v_full, bars.v_empty);
                if (*s_abort) {
                    for (int j = max(0, issued - C::NS); j < issued; ++j)
                        mbar_wait(bars.v_full + j % C::NS, (j / C::NS) & 1);
                }
            }
        } else if (lane == 0) {
            int issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int st = j % C::NS;
                if (*s_abort) break;
                if (!mbar_wait(bars.v_empty + st, ((j / C::NS) & 1) ^ 1)) { abort_cta(); break; }
                uint8_t *sv = smem + C::OFF_V + st * C::KV_BYTES;
                mbar_arrive_expect_tx(bars.v_full + st, C::KV_BYTES);
#pragma unroll
                for (int h = 0; h < C::HALVES; ++h) {
                    if (stream_once)
                        tma_load_2d_hint(sv + h * C::BOX_BYTES, &tm_v, bars.v_full + st, h * 64, kv_row0 + j * C::BN, kv_pol);
                    else
                        tma_load_2d(sv + h * C::BOX_BYTES, &tm_v, bars.v_full + st, h * 64, kv_row0 + j * C::BN);
                }
                issued = j + 1;
            }
            if (*s_abort) {
                for (int j = max(0, issued - C::NS); j < issued; ++j)
                    mbar_wait(bars.v_full + j % C::NS, (j / C::NS) & 1);
            }
        }
        __syncwarp();
        if (last_valid < C::BN) {
            // Keys past L_b may hold anything (even NaN): once the last V tile
            // has landed, zero its rows past L_b so that P = 0 really adds
            // nothing, then hand the tile to the MMA warp through v_tail.
            const int j = n_tiles - 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(bars.v_full + j % C::NS, (j / C::NS) & 1));
            if (ok) {
                uint8_t *sv = smem + C::OFF_V + (j % C::NS) * C::KV_BYTES;
                const int per_row = C::HALVES * 8;   // 16-byte chunks per key row
                for (int idx = lane; idx < (C::BN - last_valid) * per_row; idx += 32) {
                    const int r = last_valid + idx / per_row;
                    const int h = (idx % per_row) / 8, c = idx % 8;
                    *reinterpret_cast<uint4 *>(sv + h * C::BOX_BYTES + r * 128 + c * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.v_tail);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA
        regs_dec<kRegsOther>();
        // One thread issues every MMA.  The tensor pipe queues little work,
        // so each stall of this thread between MMA groups shows up as a pipe
        // bubble; the loop therefore makes all of a tile's waits at one
        // point and then issues P*V of tile j and Q K^T of tile j+2 back to
        // back (16 MMAs).  Order: QK_0, QK_1, [PV_0, QK_2], [PV_1, QK_3], ...
        // QK_{j+2} reuses S[j%2], whose P is read by PV_j just before it in
        // issue order (the pipe executes in issue order).
        if (lane == 0) {
            const uint64_t qdesc0 = smem_desc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
            const uint32_t sk0 = smem_u32(smem + C::OFF_K), sv0 = smem_u32(smem + C::OFF_V);
            const uint64_t kdesc0 = smem_desc_sw128(sk0, 16, 1024);
            const uint64_t vdesc0 = smem_desc_sw128(sv0, C::BOX_BYTES, 1024);
            auto issue_qk = [=](int j) {
                const int st = j % C::NS, g = j & 1;
                const uint64_t kd = kdesc0 + ((st * C::KV_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
                    mma_ss(tmem + C::COL_S + g * 128, qdesc0 + (off >> 4), kd + (off >> 4),
                           C::IDESC_QK, kk > 0 ? 1u : 0u);
                }
                mma_commit(bars.k_empty + st);
                mma_commit(bars.s_full + g);
            };
            auto issue_pv = [=](int jj) {
                const int st = jj % C::NS, g = jj & 1;
                const uint64_t vd = vdesc0 + ((st * C::KV_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    // P of keys 16kk..16kk+15 sits in columns 8kk..8kk+7 of S[g]
                    mma_ts(tmem + C::COL_O + g * D, tmem + C::COL_S + g * 128 + kk * 8,
                           vd + ((kk * 16 * 128) >> 4), C::IDESC_PV, (jj > 1 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bars.v_empty + st);
                if (jj == n_tiles - 1) mma_commit(bars.o_final);
            };
            bool ok = mbar_wait(bars.q_full, 0);
            for (int j = 0; ok && j < min(2, n_tiles); ++j) {
                if (!mbar_wait(bars.k_full + j % C::NS, (j / C::NS) & 1)) { ok = false; break; }
                tc_fence_after();
                issue_qk(j);
            }
            for (int jj = 0; ok && jj < n_tiles; ++jj) {
                const int st = jj % C::NS;
                const bool tail = (jj == n_tiles - 1) && last_valid < C::BN;
                const int jn = jj + 2;   // the QK that follows PV_jj in issue order
                // the three barriers are probed back to back before any wait
                uint64_t *bv = tail ? bars.v_tail : bars.v_full + st;
                const uint32_t pv = tail ? 0u : (jj / C::NS) & 1;
                uint64_t *bk_ = bars.k_full + (jn < n_tiles ? jn % C::NS : 0);
                const uint32_t pk = (jn / C::NS) & 1;
                const bool r1 = mbar_test(smem_u32(bv), pv);
                const bool r2 = mbar_test(smem_u32(bars.p_ready + (jj & 1)), (jj >> 1) & 1);
                const bool r3 = jn >= n_tiles || mbar_test(smem_u32(bk_), pk);
                if (!(r1 && r2 && r3) &&
                    (!mbar_wait(bv, pv) || !mbar_wait(bars.p_ready + (jj & 1), (jj >> 1) & 1) ||
                     (jn < n_tiles && !mbar_wait(bk_, pk)))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_pv(jj);
                if (jn < n_tiles) issue_qk(jn);
            }
            if (!ok) abort_cta();
            // every MMA this thread issued must be complete before TMEM is freed
            mma_commit(bars.drain);
            mbar_wait(bars.drain, 0);
        }
        __syncwarp();
    } else if (warp >= kFirstSoftmaxWarp) {
        // ------------------------------------------------------- softmax
        regs_inc<kRegsSoftmax>();
        const int grp = (warp - kFirstSoftmaxWarp) >> 2, wq = warp & 3;
        const int r = wq * 32 + lane;                       // row of the tile = TMEM lane
        const bool warp_active = row0 + wq * 32 < p.M;      // any real row in this warp
        const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t t_s = tmem + lane_addr + C::COL_S + grp * 128;   // this row's S/P
        const uint32_t t_o = tmem + lane_addr + C::COL_O + grp * D;     // this row's O[grp]
        const float c2 = p.scale_log2;
        bool ok = true;

        // sliding window: the first context position this row sees, L_b + d - W
        // for its node's depth d (the parent walk is bounded and overlaps the
        // first tile's loads; a bad parent array is reported by the tree
        // pass, which writes the row as NaN)
        int lo_row = 0;
        if constexpr (WINDOW) {
            const int rr = row0 + r;
            if (rr < p.M) {
                const int32_t *par = p.parent + static_cast<size_t>(b) * p.T;
                int node = rr % p.T, d = 1;
                for (int s = 0; s < p.T; ++s) {
                    const int up = par[node];
                    if (up < 0 || up >= node) break;
                    node = up;
                    ++d;
                }
                lo_row = L + d - p.window;
            }
        }
        float m_run = -INFINITY;      // running max of the scaled log2 scores (possibly stale)
        uint64_t l_exact = 0;         // pair of fp32 partial sums of 2^(x - m_run)
        uint64_t l_round = 0;         // the same over the bf16-rounded P that P*V uses
        for (int j = grp, it = 0; j < n_tiles; j += 2, ++it) {
            if (ok && !warp_wait(bars.s_full + grp, it & 1)) { ok = false; abort_cta(); }
            tc_fence_after();
            if (ok && warp_active) {
                const int n_valid = (j == n_tiles - 1) ? last_valid : C::BN;
                // the whole row (128 scores) in one batch of loads
                uint32_t r0[32], r1[32], r2[32], r3[32];
                tmem_ld32(t_s + 0, r0);
                tmem_ld32(t_s + 32, r1);
                tmem_ld32(t_s + 64, r2);
                tmem_ld32(t_s + 96, r3);
                tmem_wait_ld();
                if (n_valid < C::BN) {
                    const uint32_t ninf = __float_as_uint(-INFINITY);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        r0[i] = (i < n_valid) ? r0[i] : ninf;
                        r1[i] = (32 + i < n_valid) ? r1[i] : ninf;
                        r2[i] = (64 + i < n_valid) ? r2[i] : ninf;
                        r3[i] = (96 + i < n_valid) ? r3[i] : ninf;
                    }
                }
                if constexpr (WINDOW) {
                    // columns before this row's window (older than W - d positions)
                    const int n_lo = lo_row - (key_begin + j * C::BN);
                    if (n_lo > 0) {
                        const uint32_t ninf = __float_as_uint(-INFINITY);
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            r0[i] = (i < n_lo) ? ninf : r0[i];
                            r1[i] = (32 + i < n_lo) ? ninf : r1[i];
                            r2[i] = (64 + i < n_lo) ? ninf : r2[i];
                            r3[i] = (96 + i < n_lo) ? ninf : r3[i];
                        }
                    }
                }
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    m4[0] = max3(m4[0], __uint_as_float(r0[i]), __uint_as_float(r0[i + 1]));
                    m4[1] = max3(m4[1], __uint_as_float(r1[i]), __uint_as_float(r1[i + 1]));
                    m4[2] = max3(m4[2], __uint_as_float(r2[i]), __uint_as_float(r2[i + 1]));
                    m4[3] = max3(m4[3], __uint_as_float(r3[i]), __uint_as_float(r3[i + 1]));
                }
                const float mt = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
                const float m_new = fmaxf(m_run, mt * c2);
                bool resc = false;
                float alpha = 1.f;
                if (m_new > m_run + 8.f) {                   // lazy update
                    alpha = ex2(m_run - m_new);              // 0 on the group's first tile
                    const uint64_t aa = f2(alpha, alpha);
                    l_exact = fma2(l_exact, aa, 0ull);
                    l_round = fma2(l_round, aa, 0ull);
                    resc = it > 0;
                    m_run = m_new;
                }
                // P for the 128 keys, written as bf16 pairs over the first 64
                // score columns, 32 scores at a time
                const float mu = (m_run == -INFINITY) ? 0.f : m_run;
                const uint64_t cc = f2(c2, c2), nm = f2(-mu, -mu);
                auto exps = [&](const uint32_t (&sc)[32], int col) {
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const uint64_t x2 = fma2(f2(__uint_as_float(sc[2 * k]), __uint_as_float(sc[2 * k + 1])),
                                                 cc, nm);
                        float p0, p1;
                        constexpr int kEvery = HTA_EXP2_POLY_EVERY;   // default: one pair in four
                        if (kEvery > 0 && k % kEvery == kEvery - 1) {   // this pair on the FMA pipe
                            const float2 e = exp2_poly2(x2);
                            p0 = e.x;
                            p1 = e.y;
                        } else {
                            const float2 x = unf2(x2);
                            p0 = ex2(x.x);
                            p1 = ex2(x.y);
                        }
                        pk[k] = pack_bf16x2(p0, p1);
                        l_exact = add2(l_exact, f2(p0, p1));
                        l_round = add2(l_round, f2(bf16_lo(pk[k]), bf16_hi(pk[k])));
                    }
                    tmem_st16(t_s + col, pk);
                };
                exps(r0, 0);
                exps(r1, 16);
                exps(r2, 32);
                exps(r3, 48);
                if (__any_sync(0xffffffffu, resc)) {
                    // S of this tile was committed after P*V of the group's
                    // previous tile was issued, so O[grp] is complete here, and
                    // P*V of this tile waits for this warp's arrival below
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
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.p_ready + grp);
        }

        // ------------------------------------------------------ epilogue
        // the partials are read back by the merge right after this grid:
        // kept in L2 ahead of the K/V lines
        const uint64_t part_pol = l2_policy_evict_last();
        if (ok && !warp_wait(bars.o_final, 0)) { ok = false; abort_cta(); }
        tc_fence_after();
        // merge the two groups' online softmaxes row by row (the lse merge
        // of two KV ranges): m = max(m_0, m_1), a_g = 2^(m_g - m),
        // O = (a_0 O_0 + a_1 O_1) / (a_0 l_0 + a_1 l_1)
        float *xch = reinterpret_cast<float *>(smem + C::OFF_XCH);   // [grp][m|le|lr][row]
        {
            const float2 le = unf2(l_exact), lr = unf2(l_round);
            xch[(grp * 3 + 0) * 128 + r] = m_run;
            xch[(grp * 3 + 1) * 128 + r] = le.x + le.y;
            xch[(grp * 3 + 2) * 128 + r] = lr.x + lr.y;
        }
        const bool failed = named_bar_or(1, 256, !ok || *s_abort);
        const float m0 = xch[0 * 128 + r], m1 = xch[3 * 128 + r];
        const float m = fmaxf(m0, m1);
        const float a0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - m);
        const float a1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - m);   // group 1 had no tile
        const float l_ex = a0 * xch[1 * 128 + r] + a1 * xch[4 * 128 + r];
        const float l_rd = a0 * xch[2 * 128 + r] + a1 * xch[5 * 128 + r];
        const int rr = row0 + r;
        if (!failed) {
            // this group's half of the columns, normalised, into the staging
            // tile (16-byte chunks of a row XOR-swizzled by row % 8)
            const float inv = 1.f / l_rd;
            const float c0 = a0 * inv, c1 = a1 * inv;
            const bool has1 = n_tiles > 1;
            float *stage = reinterpret_cast<float *>(smem + C::OFF_STAGE);
            const uint32_t t_o0 = tmem + lane_addr + C::COL_O, t_o1 = t_o0 + D;
            if (warp_active) {
#pragma unroll 1
                for (int c = grp * (D / 2); c < (grp + 1) * (D / 2); c += 32) {
                    uint32_t x0[32], x1[32];
                    tmem_ld32(t_o0 + c, x0);
                    if (has1) tmem_ld32(t_o1 + c, x1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 v;
                        v.x = __uint_as_float(x0[i + 0]) * c0;
                        v.y = __uint_as_float(x0[i + 1]) * c0;
                        v.z = __uint_as_float(x0[i + 2]) * c0;
                        v.w = __uint_as_float(x0[i + 3]) * c0;
                        if (has1) {
                            v.x = fmaf(__uint_as_float(x1[i + 0]), c1, v.x);
                            v.y = fmaf(__uint_as_float(x1[i + 1]), c1, v.y);
                            v.z = fmaf(__uint_as_float(x1[i + 2]), c1, v.z);
                            v.w = fmaf(__uint_as_float(x1[i + 3]), c1, v.w);
                        }
                        const int q = (c + i) >> 2;          // 16-byte chunk of the row
                        *reinterpret_cast<float4 *>(stage + r * D + ((q ^ (r & 7)) << 2)) = v;
                    }
                }
            }
            named_bar_sync(1, 256);
            // coalesced copy-out: a row of o_part is D contiguous floats
            constexpr int CH = D / 4;                 // chunks per row
            constexpr int RPI = 32 / CH;              // rows per warp per iteration
            const int sw = warp - kFirstSoftmaxWarp;  // softmax warp 0..7
#pragma unroll 1
            for (int base = sw * RPI; base < C::BM; base += 8 * RPI) {
                const int R = base + lane / CH, q = lane % CH;
                if (row0 + R < p.M) {
                    const float4 v = *reinterpret_cast<const float4 *>(stage + R * D + ((q ^ (R & 7)) << 2));
                    st_v4_hint(p.o_part + ((grow0 + R) * p.S + split) * D + q * 4, v, part_pol);
                }
            }
        }
        if (grp == 0 && warp_active && rr < p.M)
            st_f32_hint(p.lse_part + (grow0 + r) * p.S + split, failed ? nan : (m + lg2(l_ex)) * kLn2, part_pol);
    }

    else {
        regs_dec<kRegsOther>();   // warp 3: only completes the warpgroup
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D, bool PAGED, bool WINDOW>
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
        e = cudaFuncSetAttribute(prefix_tc_kernel<D, PAGED, WINDOW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_ALLOC);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < kMaxDev) attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(p.m_tiles, p.S, p.B * p.Hkv);
    cfg.blockDim = dim3(kThreadsTc);
    cfg.dynamicSmemBytes = C::SMEM_ALLOC;
    cfg.stream = stream;
    // the launch overlaps the tail of the previous kernel on the stream; the
    // kernel's first instruction waits for that kernel to complete
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefix_tc_kernel<D, PAGED, WINDOW>, tm_q, tm_k, tm_v, p);
}

cudaError_t launch_prefix_tc(const PrefixParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                             const CUtensorMap &tm_v, cudaStream_t stream) {
    const bool paged = p.block_table != nullptr;
    if (p.window > 0)
        return p.D == 128 ? launch_tc<128, false, true>(p, tm_q, tm_k, tm_v, stream)
                          : launch_tc<64, false, true>(p, tm_q, tm_k, tm_v, stream);
    if (p.D == 128)
        return paged ? launch_tc<128, true, false>(p, tm_q, tm_k, tm_v, stream)
                     : launch_tc<128, false, false>(p, tm_q, tm_k, tm_v, stream);
    return paged ? launch_tc<64, true, false>(p, tm_q, tm_k, tm_v, stream)
                 : launch_tc<64, false, false>(p, tm_q, tm_k, tm_v, stream);
}

}  // namespace hta
