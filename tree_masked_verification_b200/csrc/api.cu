// api.cu -- the C ABI of liblongspec_hta.so (declared in include/longspec_hta.h).
//
// Host side only: argument checks, the split-KV chunking, tensor-map
// (TMA descriptor) encoding with a small per-pointer cache, and the two
// launches of one verification call (prefix kernel, then the tree pass fused
// with the log-sum-exp merge).  Nothing here computes attention.
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/longspec_hta.h"
#include "hta_kernels.h"

using hta::PrefixParams;
using hta::TreeMergeParams;

namespace {

// ---------------------------------------------------------------- device
struct DeviceInfo {
    bool probed = false;
    bool supported = false;
    int num_sms = 0;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device(DeviceInfo *out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LONGSPEC_HTA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return LONGSPEC_HTA_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.probed) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return LONGSPEC_HTA_ERR_CUDA;
        d.supported = (major == 10 && minor == 0);
        d.num_sms = sms;
        d.probed = true;
    }
    *out = d;
    return d.supported ? LONGSPEC_HTA_OK : LONGSPEC_HTA_ERR_UNSUPPORTED_DEVICE;
}

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

struct MapKey {
    int dev;
    const void *ptr;
    uint64_t rows;
    int D;
    int box_rows;
    bool operator==(const MapKey &o) const {
        return dev == o.dev && ptr == o.ptr && rows == o.rows && D == o.D && box_rows == o.box_rows;
    }
};
struct MapEntry {
    MapKey key;
    CUtensorMap map;
    bool used;
};
constexpr int kMapCache = 48;
MapEntry g_maps[kMapCache];
int g_map_next = 0;
std::mutex g_map_mu;

// [rows][D] bf16 matrix as 64-column x box_rows-row boxes with 128-byte
// swizzle (box_rows 128 for Q and contiguous K/V, the block size for a
// paged cache).
int tensor_map(const void *ptr, uint64_t rows, int D, CUtensorMap *out, int box_rows = 128) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LONGSPEC_HTA_ERR_CUDA;
    const MapKey key{dev, ptr, rows, D, box_rows};
    std::lock_guard<std::mutex> lk(g_map_mu);
    for (auto &e : g_maps)
        if (e.used && e.key == key) { *out = e.map; return LONGSPEC_HTA_OK; }
    EncodeTiledFn fn = encode_fn();
    if (!fn) return LONGSPEC_HTA_ERR_CUDA;
    CUtensorMap m;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), rows};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return LONGSPEC_HTA_ERR_CUDA;
    MapEntry &e = g_maps[g_map_next];
    g_map_next = (g_map_next + 1) % kMapCache;
    e.key = key;
    e.map = m;
    e.used = true;
    *out = m;
    return LONGSPEC_HTA_OK;
}

// ------------------------------------------------------------- validation
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const longspec_hta_dims *d) {
    if (!d) return LONGSPEC_HTA_ERR_NULL_POINTER;
    if (d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->T < 1 || d->L_cap < 0 || d->Hq % d->Hkv != 0)
        return LONGSPEC_HTA_ERR_INVALID_DIMS;
    if (!(d->scale >= 0.f) || std::isinf(d->scale)) return LONGSPEC_HTA_ERR_INVALID_DIMS;
    if (d->D != 64 && d->D != 128) return LONGSPEC_HTA_ERR_UNSUPPORTED_D;
    if (d->T > LONGSPEC_HTA_T_MAX) return LONGSPEC_HTA_ERR_T_TOO_LARGE;
    const long long rows = 1LL * d->B * d->Hq * d->T;
    const long long keys = 1LL * d->B * d->Hkv * d->L_cap;
    if (rows >= (1LL << 31) || keys + 128 >= (1LL << 31) || 1LL * d->B * d->Hkv > 65535)
        return LONGSPEC_HTA_ERR_INVALID_DIMS;
    return LONGSPEC_HTA_OK;
}

float scale_of(const longspec_hta_dims *d) {
    return d->scale > 0.f ? d->scale : 1.f / std::sqrt(static_cast<float>(d->D));
}

int m_tiles_of(const longspec_hta_dims *d) {
    const int M = (d->Hq / d->Hkv) * d->T;
    return (M + 127) / 128;
}

// Split-KV chunking: chunk_tiles tiles of 128 keys per split, S splits.
struct Chunking {
    int S, chunk_tiles;
};

Chunking chunking_for(const longspec_hta_dims *d, int requested, int num_sms) {
    const int tiles = std::max(1, (d->L_cap + hta::kKeyTile - 1) / hta::kKeyTile);
    auto make = [&](int s) {
        s = std::max(1, std::min(std::min(s, tiles), hta::kMaxSplits));
        const int ct = (tiles + s - 1) / s;
        return Chunking{(tiles + ct - 1) / ct, ct};
    };
    if (requested > 0) return make(requested);
    // smallest estimated time: waves of CTAs x (tiles per CTA + fixed cost)
    const long long units = 1LL * d->B * d->Hkv * m_tiles_of(d);
    Chunking best = make(1);
    double best_cost = 1e300;
    for (int s = 1; s <= std::min(tiles, hta::kMaxSplits); ++s) {
        const Chunking c = make(s);
        const long long ctas = units * c.S;
        const long long waves = (ctas + num_sms - 1) / std::max(1, num_sms);
        const double cost = waves * (c.chunk_tiles + 2.0) + 0.05 * c.S;
        if (cost < best_cost - 1e-9) { best_cost = cost; best = c; }
    }
    return best;
}

struct WsLayout {
    size_t o_off, lse_off, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

WsLayout ws_layout(const longspec_hta_dims *d, int S) {
    const size_t rows = 1ull * d->B * d->Hq * d->T;
    WsLayout w;
    w.o_off = hta::kStatusBytes;
    w.lse_off = align256(w.o_off + rows * S * d->D * sizeof(float));
    w.total = align256(w.lse_off + rows * S * sizeof(float));
    return w;
}

PrefixParams prefix_params(const longspec_hta_dims *d, const Chunking &c, const void *q,
                           const void *kp, const void *vp, const int32_t *plen, float *o_part,
                           float *lse_part, uint32_t *status) {
    PrefixParams p{};
    p.B = d->B; p.Hq = d->Hq; p.Hkv = d->Hkv; p.D = d->D; p.T = d->T; p.L_cap = d->L_cap;
    p.G = d->Hq / d->Hkv;
    p.M = p.G * d->T;
    p.m_tiles = (p.M + 127) / 128;
    p.S = c.S;
    p.chunk_tiles = c.chunk_tiles;
    p.scale_log2 = scale_of(d) * hta::kLog2e;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k_prefix = static_cast<const __nv_bfloat16 *>(kp);
    p.v_prefix = static_cast<const __nv_bfloat16 *>(vp);
    p.prefix_len = plen;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.status = status;
    return p;
}

int run_prefix(const longspec_hta_dims *d, const PrefixParams &p, int kernel, cudaEvent_t ev_begin,
               cudaEvent_t ev_end, cudaStream_t stream) {
    CUtensorMap tq, tk, tv;
    const bool tc = kernel == LONGSPEC_HTA_PREFIX_TCGEN05;
    if (tc) {
        const uint64_t qrows = 1ull * d->B * d->Hq * d->T;
        const bool paged = p.block_table != nullptr;
        const uint64_t krows = paged ? 1ull * p.num_blocks * d->Hkv * p.block_size
                                     : 1ull * d->B * d->Hkv * std::max(d->L_cap, 1);
        const int box = paged ? p.block_size : 128;
        int rc;
        if ((rc = tensor_map(p.q, qrows, d->D, &tq)) != LONGSPEC_HTA_OK) return rc;
        if ((rc = tensor_map(p.k_prefix, krows, d->D, &tk, box)) != LONGSPEC_HTA_OK) return rc;
        if ((rc = tensor_map(p.v_prefix, krows, d->D, &tv, box)) != LONGSPEC_HTA_OK) return rc;
    }
    if (ev_begin && cudaEventRecord(ev_begin, stream) != cudaSuccess) return LONGSPEC_HTA_ERR_CUDA;
    cudaError_t e = tc ? hta::launch_prefix_tc(p, tq, tk, tv, stream) : hta::launch_prefix_simt(p, stream);
    if (e != cudaSuccess) return LONGSPEC_HTA_ERR_CUDA;
    if (ev_end && cudaEventRecord(ev_end, stream) != cudaSuccess) return LONGSPEC_HTA_ERR_CUDA;
    return LONGSPEC_HTA_OK;
}

TreeMergeParams tree_params(const longspec_hta_dims *d, int mode, int S, const void *q,
                            const void *kt, const void *vt, const int32_t *parent,
                            const int32_t *plen, const float *o_part, const float *lse_part,
                            uint32_t *status) {
    TreeMergeParams t{};
    t.B = d->B; t.Hq = d->Hq; t.Hkv = d->Hkv; t.D = d->D; t.T = d->T; t.L_cap = d->L_cap;
    t.S = S;
    t.scale_log2 = scale_of(d) * hta::kLog2e;
    t.mode = mode;
    t.q = static_cast<const __nv_bfloat16 *>(q);
    t.k_tree = static_cast<const __nv_bfloat16 *>(kt);
    t.v_tree = static_cast<const __nv_bfloat16 *>(vt);
    t.parent = parent;
    t.prefix_len = plen;
    t.o_part = o_part;
    t.lse_part = lse_part;
    t.status = status;
    return t;
}

}  // namespace

extern "C" {

int longspec_hta_abi_version(void) { return LONGSPEC_HTA_ABI_VERSION; }

#define HTA_STR2(x) #x
#define HTA_STR(x) HTA_STR2(x)
const char *longspec_hta_build_info(void) {
    return "kv_stages_d128=" HTA_STR(HTA_KV_STAGES_D128) " exp2_poly_every=" HTA_STR(HTA_EXP2_POLY_EVERY);
}

const char *longspec_hta_strerror(int code) {
    switch (code) {
    case LONGSPEC_HTA_OK: return "ok";
    case LONGSPEC_HTA_ERR_INVALID_DIMS: return "invalid dimensions or scale";
    case LONGSPEC_HTA_ERR_NULL_POINTER: return "null pointer";
    case LONGSPEC_HTA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case LONGSPEC_HTA_ERR_T_TOO_LARGE: return "tree larger than LONGSPEC_HTA_T_MAX";
    case LONGSPEC_HTA_ERR_UNSUPPORTED_D: return "head dimension must be 64 or 128";
    case LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case LONGSPEC_HTA_ERR_CUDA: return "CUDA call failed";
    case LONGSPEC_HTA_ERR_UNSUPPORTED_DEVICE: return "current device is not sm_100 (B200)";
    case LONGSPEC_HTA_ERR_INVALID_OPTION: return "invalid option";
    case LONGSPEC_HTA_ERR_BAD_PARENT: return "parent[i] outside [-1, i)";
    case LONGSPEC_HTA_ERR_PREFIX_LEN_RANGE: return "prefix_len outside [0, L_cap]";
    case LONGSPEC_HTA_ERR_PIPELINE_TIMEOUT: return "in-kernel wait timed out";
    case LONGSPEC_HTA_ERR_INTERNAL: return "internal kernel precondition failed";
    case LONGSPEC_HTA_ERR_BAD_BLOCK: return "a block_table entry is outside [0, num_blocks)";
    case LONGSPEC_HTA_ERR_BAD_PATH: return "an accepted length or path entry is out of range";
    default: return "unknown status";
    }
}

int longspec_hta_default_splits(const longspec_hta_dims *dims) {
    int rc = check_dims(dims);
    if (rc) return rc;
    DeviceInfo di;
    rc = current_device(&di);
    if (rc) return rc;
    return chunking_for(dims, 0, di.num_sms).S;
}

int longspec_hta_chunking(const longspec_hta_dims *dims, int num_splits, int *num_splits_out,
                          int *chunk_keys_out) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (num_splits < 0) return LONGSPEC_HTA_ERR_INVALID_OPTION;
    int sms = 148;
    if (num_splits == 0) {
        DeviceInfo di;
        if ((rc = current_device(&di))) return rc;
        sms = di.num_sms;
    }
    const Chunking c = chunking_for(dims, num_splits, sms);
    if (num_splits_out) *num_splits_out = c.S;
    if (chunk_keys_out) *chunk_keys_out = c.chunk_tiles * hta::kKeyTile;
    return LONGSPEC_HTA_OK;
}

size_t longspec_hta_workspace_bytes(const longspec_hta_dims *dims, int num_splits) {
    if (check_dims(dims) != LONGSPEC_HTA_OK || num_splits < 0) return 0;
    int sms = 148;
    if (num_splits == 0) {
        DeviceInfo di;
        if (current_device(&di) != LONGSPEC_HTA_OK) return 0;
        sms = di.num_sms;
    }
    return ws_layout(dims, chunking_for(dims, num_splits, sms).S).total;
}

int longspec_hta_workspace_init(void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!workspace) return LONGSPEC_HTA_ERR_NULL_POINTER;
    if (!aligned16(workspace)) return LONGSPEC_HTA_ERR_MISALIGNED;
    if (workspace_bytes < static_cast<size_t>(hta::kStatusBytes)) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    return cudaMemsetAsync(workspace, 0, hta::kStatusBytes, stream) == cudaSuccess ? LONGSPEC_HTA_OK
                                                                                  : LONGSPEC_HTA_ERR_CUDA;
}

// One verification call (prefix_only = false) or prefix-only attention
// (prefix_only = true), the prefix K/V contiguous (kv == nullptr) or paged.
static int run_attention(const longspec_hta_dims *dims, const void *q, const void *k_prefix,
                         const void *v_prefix, const longspec_hta_paged_kv *kv,
                         const int32_t *prefix_len, const void *k_tree, const void *v_tree,
                         const int32_t *parent, void *out, float *lse, void *workspace,
                         size_t workspace_bytes, const longspec_hta_options *opts,
                         cudaStream_t stream, bool prefix_only) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (kv) {
        k_prefix = kv->k_cache;
        v_prefix = kv->v_cache;
        if (!kv->block_table) return LONGSPEC_HTA_ERR_NULL_POINTER;
        if ((reinterpret_cast<uintptr_t>(kv->block_table) & 3u) != 0) return LONGSPEC_HTA_ERR_MISALIGNED;
    }
    const void *ptrs[] = {q, k_prefix, v_prefix, prefix_len, out, lse, workspace,
                          prefix_only ? q : k_tree, prefix_only ? q : v_tree, prefix_only ? q : parent};
    for (const void *p : ptrs) {
        if (!p) return LONGSPEC_HTA_ERR_NULL_POINTER;
        if (!aligned16(p)) return LONGSPEC_HTA_ERR_MISALIGNED;
    }
    if (kv) {
        const int bs = kv->block_size;
        if ((bs != 16 && bs != 32 && bs != 64 && bs != 128) || kv->num_blocks < 1 || kv->max_blocks < 1 ||
            1LL * kv->max_blocks * bs < dims->L_cap ||
            1LL * kv->num_blocks * dims->Hkv * bs + 128 >= (1LL << 31))
            return LONGSPEC_HTA_ERR_INVALID_DIMS;
    }
    longspec_hta_options o{};
    if (opts) o = *opts;
    if (o.num_splits < 0 || (o.prefix_kernel != LONGSPEC_HTA_PREFIX_TCGEN05 &&
                             o.prefix_kernel != LONGSPEC_HTA_PREFIX_SIMT) ||
        (kv && o.prefix_kernel == LONGSPEC_HTA_PREFIX_SIMT))
        return LONGSPEC_HTA_ERR_INVALID_OPTION;
    DeviceInfo di;
    if ((rc = current_device(&di))) return rc;
    const Chunking c = chunking_for(dims, o.num_splits, di.num_sms);
    const WsLayout w = ws_layout(dims, c.S);
    if (workspace_bytes < w.total) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    float *o_part = reinterpret_cast<float *>(ws + w.o_off);
    float *lse_part = reinterpret_cast<float *>(ws + w.lse_off);

    PrefixParams pp = prefix_params(dims, c, q, k_prefix, v_prefix, prefix_len, o_part, lse_part, status);
    if (kv) {
        pp.block_table = kv->block_table;
        pp.block_size = kv->block_size;
        pp.max_blocks = kv->max_blocks;
        pp.num_blocks = kv->num_blocks;
    }
    if ((rc = run_prefix(dims, pp, o.prefix_kernel, o.prefix_begin, o.prefix_end, stream))) return rc;
    TreeMergeParams tp = prefix_only
        ? tree_params(dims, hta::kTreeModePrefixOnly, c.S, q, nullptr, nullptr, nullptr, prefix_len,
                      o_part, lse_part, status)
        : tree_params(dims, hta::kTreeModeMerge, c.S, q, k_tree, v_tree, parent, prefix_len, o_part,
                      lse_part, status);
    tp.out = static_cast<__nv_bfloat16 *>(out);
    tp.lse = lse;
    return hta::launch_tree_merge(tp, stream) == cudaSuccess ? LONGSPEC_HTA_OK : LONGSPEC_HTA_ERR_CUDA;
}

int longspec_hta_verify_ex(const longspec_hta_dims *dims, const void *q, const void *k_prefix,
                           const void *v_prefix, const int32_t *prefix_len, const void *k_tree,
                           const void *v_tree, const int32_t *parent, void *out, float *lse,
                           void *workspace, size_t workspace_bytes,
                           const longspec_hta_options *opts, cudaStream_t stream) {
    return run_attention(dims, q, k_prefix, v_prefix, nullptr, prefix_len, k_tree, v_tree, parent, out,
                         lse, workspace, workspace_bytes, opts, stream, false);
}

int longspec_hta_verify_paged(const longspec_hta_dims *dims, const void *q, const longspec_hta_paged_kv *kv,
                              const int32_t *prefix_len, const void *k_tree, const void *v_tree,
                              const int32_t *parent, void *out, float *lse, void *workspace,
                              size_t workspace_bytes, const longspec_hta_options *opts,
                              cudaStream_t stream) {
    if (!kv) return LONGSPEC_HTA_ERR_NULL_POINTER;
    return run_attention(dims, q, nullptr, nullptr, kv, prefix_len, k_tree, v_tree, parent, out, lse,
                         workspace, workspace_bytes, opts, stream, false);
}

int longspec_hta_verify(const longspec_hta_dims *dims, const void *q, const void *k_prefix,
                        const void *v_prefix, const int32_t *prefix_len, const void *k_tree,
                        const void *v_tree, const int32_t *parent, void *out, float *lse,
                        void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    return longspec_hta_verify_ex(dims, q, k_prefix, v_prefix, prefix_len, k_tree, v_tree, parent,
                                  out, lse, workspace, workspace_bytes, nullptr, stream);
}

// ---- end-to-end call on host buffers -------------------------------------
namespace {
struct ArenaLayout {
    size_t q, kp, vp, plen, kt, vt, par, out, lse, ws, total;
    size_t q_b, kv_b, plen_b, tree_b, par_b, out_b, lse_b, ws_b;
};

ArenaLayout arena_layout(const longspec_hta_dims *d, int num_sms) {
    ArenaLayout a{};
    a.q_b = 2ull * d->B * d->Hq * d->T * d->D;
    a.kv_b = 2ull * d->B * d->Hkv * d->L_cap * d->D;
    a.plen_b = 4ull * d->B;
    a.tree_b = 2ull * d->B * d->Hkv * d->T * d->D;
    a.par_b = 4ull * d->B * d->T;
    a.out_b = a.q_b;
    a.lse_b = 4ull * d->B * d->Hq * d->T;
    a.ws_b = ws_layout(d, chunking_for(d, 0, num_sms).S).total;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align256(off + std::max<size_t>(bytes, 1)); return o; };
    a.q = take(a.q_b); a.kp = take(a.kv_b); a.vp = take(a.kv_b); a.plen = take(a.plen_b);
    a.kt = take(a.tree_b); a.vt = take(a.tree_b); a.par = take(a.par_b);
    a.out = take(a.out_b); a.lse = take(a.lse_b); a.ws = take(a.ws_b);
    a.total = off;
    return a;
}
}  // namespace

size_t longspec_hta_host_arena_bytes(const longspec_hta_dims *dims) {
    if (check_dims(dims) != LONGSPEC_HTA_OK) return 0;
    DeviceInfo di;
    if (current_device(&di) != LONGSPEC_HTA_OK) return 0;
    return arena_layout(dims, di.num_sms).total;
}

int longspec_hta_verify_host(const longspec_hta_dims *dims, const void *q, const void *k_prefix,
                             const void *v_prefix, const int32_t *prefix_len, const void *k_tree,
                             const void *v_tree, const int32_t *parent, void *out, float *lse,
                             void *arena, size_t arena_bytes, cudaStream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    const void *ptrs[] = {q, k_prefix, v_prefix, prefix_len, k_tree, v_tree, parent, out, lse, arena};
    for (const void *p : ptrs)
        if (!p) return LONGSPEC_HTA_ERR_NULL_POINTER;
    if (!aligned16(arena)) return LONGSPEC_HTA_ERR_MISALIGNED;
    DeviceInfo di;
    if ((rc = current_device(&di))) return rc;
    const ArenaLayout a = arena_layout(dims, di.num_sms);
    if (arena_bytes < a.total) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    uint8_t *base = static_cast<uint8_t *>(arena);
    struct Copy { size_t off; const void *src; size_t bytes; };
    const Copy ins[] = {{a.q, q, a.q_b}, {a.kp, k_prefix, a.kv_b}, {a.vp, v_prefix, a.kv_b},
                        {a.plen, prefix_len, a.plen_b}, {a.kt, k_tree, a.tree_b},
                        {a.vt, v_tree, a.tree_b}, {a.par, parent, a.par_b}};
    for (const Copy &c : ins)
        if (c.bytes && cudaMemcpyAsync(base + c.off, c.src, c.bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess)
            return LONGSPEC_HTA_ERR_CUDA;
    if (cudaMemsetAsync(base + a.ws, 0, hta::kStatusBytes, stream) != cudaSuccess) return LONGSPEC_HTA_ERR_CUDA;
    rc = longspec_hta_verify(dims, base + a.q, base + a.kp, base + a.vp,
                             reinterpret_cast<const int32_t *>(base + a.plen), base + a.kt, base + a.vt,
                             reinterpret_cast<const int32_t *>(base + a.par), base + a.out,
                             reinterpret_cast<float *>(base + a.lse), base + a.ws, a.ws_b, stream);
    if (rc) return rc;
    if (cudaMemcpyAsync(out, base + a.out, a.out_b, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaMemcpyAsync(lse, base + a.lse, a.lse_b, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return LONGSPEC_HTA_ERR_CUDA;
    return LONGSPEC_HTA_OK;
}

// ---- debug exports --------------------------------------------------------
int longspec_hta_tree_mask(const int32_t *parent, int B, int T, uint32_t *bits, void *workspace,
                           size_t workspace_bytes, cudaStream_t stream) {
    if (!parent || !bits || !workspace) return LONGSPEC_HTA_ERR_NULL_POINTER;
    if (!aligned16(parent) || !aligned16(bits) || !aligned16(workspace)) return LONGSPEC_HTA_ERR_MISALIGNED;
    if (B < 1 || B > 65535 || T < 1) return LONGSPEC_HTA_ERR_INVALID_DIMS;
    if (T > LONGSPEC_HTA_T_MAX) return LONGSPEC_HTA_ERR_T_TOO_LARGE;
    if (workspace_bytes < static_cast<size_t>(hta::kStatusBytes)) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo di;
    int rc = current_device(&di);
    if (rc) return rc;
    TreeMergeParams t{};
    t.B = B; t.Hq = 1; t.Hkv = 1; t.D = 128; t.T = T;
    t.mode = hta::kTreeModeMask;
    t.parent = parent;
    t.mask_out = bits;
    t.status = static_cast<uint32_t *>(workspace);
    return hta::launch_tree_merge(t, stream) == cudaSuccess ? LONGSPEC_HTA_OK : LONGSPEC_HTA_ERR_CUDA;
}

int longspec_hta_tree_partial(const longspec_hta_dims *dims, const void *q, const void *k_tree,
                              const void *v_tree, const int32_t *parent, float *o_tree,
                              float *lse_tree, void *workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    const void *ptrs[] = {q, k_tree, v_tree, parent, o_tree, lse_tree, workspace};
    for (const void *p : ptrs) {
        if (!p) return LONGSPEC_HTA_ERR_NULL_POINTER;
        if (!aligned16(p)) return LONGSPEC_HTA_ERR_MISALIGNED;
    }
    if (workspace_bytes < static_cast<size_t>(hta::kStatusBytes)) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo di;
    if ((rc = current_device(&di))) return rc;
    TreeMergeParams t = tree_params(dims, hta::kTreeModePartial, 0, q, k_tree, v_tree, parent, nullptr,
                                    nullptr, nullptr, static_cast<uint32_t *>(workspace));
    t.o_tree = o_tree;
    t.lse_tree = lse_tree;
    return hta::launch_tree_merge(t, stream) == cudaSuccess ? LONGSPEC_HTA_OK : LONGSPEC_HTA_ERR_CUDA;
}

int longspec_hta_prefix_partial(const longspec_hta_dims *dims, const void *q, const void *k_prefix,
                                const void *v_prefix, const int32_t *prefix_len, float *o_part,
                                float *lse_part, int num_splits, int prefix_kernel,
                                int *num_splits_out, void *workspace, size_t workspace_bytes,
                                cudaStream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    const void *ptrs[] = {q, k_prefix, v_prefix, prefix_len, o_part, lse_part, workspace};
    for (const void *p : ptrs) {
        if (!p) return LONGSPEC_HTA_ERR_NULL_POINTER;
        if (!aligned16(p)) return LONGSPEC_HTA_ERR_MISALIGNED;
    }
    if (num_splits < 0 || (prefix_kernel != LONGSPEC_HTA_PREFIX_TCGEN05 &&
                           prefix_kernel != LONGSPEC_HTA_PREFIX_SIMT))
        return LONGSPEC_HTA_ERR_INVALID_OPTION;
    if (workspace_bytes < static_cast<size_t>(hta::kStatusBytes)) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo di;
    if ((rc = current_device(&di))) return rc;
    const Chunking c = chunking_for(dims, num_splits, di.num_sms);
    if (num_splits_out) *num_splits_out = c.S;
    const PrefixParams pp = prefix_params(dims, c, q, k_prefix, v_prefix, prefix_len, o_part, lse_part,
                                          static_cast<uint32_t *>(workspace));
    return run_prefix(dims, pp, prefix_kernel, nullptr, nullptr, stream);
}

int longspec_hta_prefix_attention(const longspec_hta_dims *dims, const void *q, const void *k_prefix,
                                  const void *v_prefix, const int32_t *prefix_len, void *out, float *lse,
                                  void *workspace, size_t workspace_bytes,
                                  const longspec_hta_options *opts, cudaStream_t stream) {
    return run_attention(dims, q, k_prefix, v_prefix, nullptr, prefix_len, nullptr, nullptr, nullptr, out,
                         lse, workspace, workspace_bytes, opts, stream, true);
}

int longspec_hta_prefix_attention_paged(const longspec_hta_dims *dims, const void *q,
                                        const longspec_hta_paged_kv *kv, const int32_t *prefix_len,
                                        void *out, float *lse, void *workspace, size_t workspace_bytes,
                                        const longspec_hta_options *opts, cudaStream_t stream) {
    if (!kv) return LONGSPEC_HTA_ERR_NULL_POINTER;
    return run_attention(dims, q, nullptr, nullptr, kv, prefix_len, nullptr, nullptr, nullptr, out, lse,
                         workspace, workspace_bytes, opts, stream, true);
}

// ---- greedy acceptance ------------------------------------------------------
namespace {
constexpr int kAcceptMaxSlices = 32;
// slices per logits row: about two CTAs per SM over the grid (measured on
// B200 against one, four, eight and sixteen: fewer, longer slices lose the
// parallelism of a short wave, more of them add CTAs whose ramp and
// reduction outweigh their share of the stream)
int accept_slices(int B, int T, int V, int num_sms) {
    const long long rows = 1LL * B * (T + 1);
    long long want = (2LL * num_sms + rows - 1) / rows;
    want = std::min<long long>(want, (V + 2047) / 2048);     // at least 2048 elements a slice
    return static_cast<int>(std::max<long long>(1, std::min<long long>(want, kAcceptMaxSlices)));
}
}  // namespace

size_t longspec_hta_accept_workspace_bytes(int B, int T, int V) {
    if (B < 1 || T < 1 || T > LONGSPEC_HTA_T_MAX || V < 1) return 0;
    const size_t rows = static_cast<size_t>(B) * (T + 1);
    return hta::kStatusBytes + rows * kAcceptMaxSlices * (sizeof(float) + sizeof(int));
}

int longspec_hta_accept_greedy(int B, int T, int V, const void *logits, const int32_t *draft_tokens,
                               const int32_t *parent, int32_t *accept_len, int32_t *path, int32_t *bonus,
                               void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (B < 1 || T < 1 || V < 1 || 1LL * B * (T + 1) > 65535 || 1LL * B * (T + 1) * V >= (1LL << 40))
        return LONGSPEC_HTA_ERR_INVALID_DIMS;
    if (T > LONGSPEC_HTA_T_MAX) return LONGSPEC_HTA_ERR_T_TOO_LARGE;
    const void *ptrs[] = {logits, draft_tokens, parent, accept_len, path, bonus, workspace};
    for (const void *q : ptrs) {
        if (!q) return LONGSPEC_HTA_ERR_NULL_POINTER;
        if ((reinterpret_cast<uintptr_t>(q) & 3u) != 0) return LONGSPEC_HTA_ERR_MISALIGNED;
    }
    if (!aligned16(logits) || !aligned16(workspace)) return LONGSPEC_HTA_ERR_MISALIGNED;
    if (workspace_bytes < longspec_hta_accept_workspace_bytes(B, T, V)) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo di;
    int rc;
    if ((rc = current_device(&di))) return rc;
    hta::AcceptParams p{};
    p.B = B; p.T = T; p.V = V;
    p.n_slices = accept_slices(B, T, V, di.num_sms);
    p.slice = ((V + p.n_slices - 1) / p.n_slices + 7) / 8 * 8;
    p.n_slices = (V + p.slice - 1) / p.slice;
    p.logits = static_cast<const __nv_bfloat16 *>(logits);
    p.draft_tokens = draft_tokens;
    p.parent = parent;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const size_t rows = static_cast<size_t>(B) * (T + 1);
    p.status = reinterpret_cast<uint32_t *>(ws);
    p.part_v = reinterpret_cast<float *>(ws + hta::kStatusBytes);
    p.part_i = reinterpret_cast<int *>(ws + hta::kStatusBytes + rows * kAcceptMaxSlices * sizeof(float));
    p.accept_len = accept_len;
    p.path = path;
    p.bonus = bonus;
    return hta::launch_accept(p, stream) == cudaSuccess ? LONGSPEC_HTA_OK : LONGSPEC_HTA_ERR_CUDA;
}

// ---- sliding-window tree attention (the draft model's self-attention) ------
namespace {
// The window spans at most W/128 + 1 key tiles (its start need not be tile
// aligned), read by one chunk: on B200 one CTA per (row tile, KV head) over
// the whole window beat splitting it (13.3 against 14.7 us per call for 32
// heads over 8 KV heads, 68 nodes, W = 512: a split adds a CTA's fixed cost
// and a partial to merge, and the window is only a few tiles long).
int window_tiles(const longspec_hta_dims *d) { return d->L_cap / hta::kKeyTile + 1; }

int check_window_dims(const longspec_hta_dims *d) {
    int rc = check_dims(d);
    if (rc) return rc;
    if (d->L_cap < 128 || d->L_cap % 128 != 0 || d->L_cap <= d->T) return LONGSPEC_HTA_ERR_INVALID_DIMS;
    return LONGSPEC_HTA_OK;
}
}  // namespace

size_t longspec_hta_window_workspace_bytes(const longspec_hta_dims *dims) {
    if (check_window_dims(dims) != LONGSPEC_HTA_OK) return 0;
    return ws_layout(dims, 1).total;
}

int longspec_hta_window_verify(const longspec_hta_dims *dims, const void *q, const void *k_ring,
                               const void *v_ring, const int32_t *prefix_len, const void *k_tree,
                               const void *v_tree, const int32_t *parent, void *out, float *lse,
                               void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    int rc = check_window_dims(dims);
    if (rc) return rc;
    const int W = dims->L_cap;
    const void *ptrs[] = {q, k_ring, v_ring, prefix_len, k_tree, v_tree, parent, out, lse, workspace};
    for (const void *p : ptrs) {
        if (!p) return LONGSPEC_HTA_ERR_NULL_POINTER;
        if (!aligned16(p)) return LONGSPEC_HTA_ERR_MISALIGNED;
    }
    DeviceInfo di;
    if ((rc = current_device(&di))) return rc;
    const Chunking c{1, window_tiles(dims)};
    const WsLayout w = ws_layout(dims, c.S);
    if (workspace_bytes < w.total) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    float *o_part = reinterpret_cast<float *>(ws + w.o_off);
    float *lse_part = reinterpret_cast<float *>(ws + w.lse_off);
    PrefixParams pp = prefix_params(dims, c, q, k_ring, v_ring, prefix_len, o_part, lse_part, status);
    pp.window = W;
    pp.parent = parent;
    if ((rc = run_prefix(dims, pp, LONGSPEC_HTA_PREFIX_TCGEN05, nullptr, nullptr, stream))) return rc;
    TreeMergeParams tp = tree_params(dims, hta::kTreeModeMerge, c.S, q, k_tree, v_tree, parent, prefix_len,
                                     o_part, lse_part, status);
    tp.window = W;
    tp.out = static_cast<__nv_bfloat16 *>(out);
    tp.lse = lse;
    return hta::launch_tree_merge(tp, stream) == cudaSuccess ? LONGSPEC_HTA_OK : LONGSPEC_HTA_ERR_CUDA;
}

// ---- KV commit of the accepted path ----------------------------------------
namespace {
int run_commit(const longspec_hta_dims *dims, void *k_cache, void *v_cache,
               const longspec_hta_paged_kv *kv, int32_t *prefix_len, const void *k_tree,
               const void *v_tree, const int32_t *accept_len, const int32_t *path, void *workspace,
               size_t workspace_bytes, cudaStream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (kv) {   // the commit writes the cache the descriptor points to
        k_cache = const_cast<void *>(kv->k_cache);
        v_cache = const_cast<void *>(kv->v_cache);
    }
    const void *big[] = {k_cache, v_cache, k_tree, v_tree, workspace};
    for (const void *q : big) {
        if (!q) return LONGSPEC_HTA_ERR_NULL_POINTER;
        if (!aligned16(q)) return LONGSPEC_HTA_ERR_MISALIGNED;
    }
    const void *ints[] = {prefix_len, accept_len, path, kv ? static_cast<const void *>(kv->block_table) : path};
    for (const void *q : ints) {
        if (!q) return LONGSPEC_HTA_ERR_NULL_POINTER;
        if ((reinterpret_cast<uintptr_t>(q) & 3u) != 0) return LONGSPEC_HTA_ERR_MISALIGNED;
    }
    if (kv) {
        const int bs = kv->block_size;
        if ((bs != 16 && bs != 32 && bs != 64 && bs != 128) || kv->num_blocks < 1 || kv->max_blocks < 1 ||
            1LL * kv->max_blocks * bs < dims->L_cap ||
            1LL * kv->num_blocks * dims->Hkv * bs + 128 >= (1LL << 31))
            return LONGSPEC_HTA_ERR_INVALID_DIMS;
    }
    if (workspace_bytes < static_cast<size_t>(hta::kStatusBytes)) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo di;
    if ((rc = current_device(&di))) return rc;
    hta::CommitParams p{};
    p.B = dims->B; p.Hkv = dims->Hkv; p.D = dims->D; p.T = dims->T; p.L_cap = dims->L_cap;
    p.k_cache = static_cast<__nv_bfloat16 *>(k_cache);
    p.v_cache = static_cast<__nv_bfloat16 *>(v_cache);
    if (kv) {
        p.block_table = kv->block_table;
        p.block_size = kv->block_size;
        p.max_blocks = kv->max_blocks;
        p.num_blocks = kv->num_blocks;
    }
    p.prefix_len = prefix_len;
    p.k_tree = static_cast<const __nv_bfloat16 *>(k_tree);
    p.v_tree = static_cast<const __nv_bfloat16 *>(v_tree);
    p.accept_len = accept_len;
    p.path = path;
    p.status = static_cast<uint32_t *>(workspace);
    return hta::launch_commit(p, stream) == cudaSuccess ? LONGSPEC_HTA_OK : LONGSPEC_HTA_ERR_CUDA;
}
}  // namespace

int longspec_hta_commit(const longspec_hta_dims *dims, void *k_prefix, void *v_prefix,
                        int32_t *prefix_len, const void *k_tree, const void *v_tree,
                        const int32_t *accept_len, const int32_t *path, void *workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
    return run_commit(dims, k_prefix, v_prefix, nullptr, prefix_len, k_tree, v_tree, accept_len, path,
                      workspace, workspace_bytes, stream);
}

int longspec_hta_commit_paged(const longspec_hta_dims *dims, const longspec_hta_paged_kv *kv,
                              int32_t *prefix_len, const void *k_tree, const void *v_tree,
                              const int32_t *accept_len, const int32_t *path, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
    if (!kv) return LONGSPEC_HTA_ERR_NULL_POINTER;
    return run_commit(dims, nullptr, nullptr, kv, prefix_len, k_tree, v_tree, accept_len, path,
                      workspace, workspace_bytes, stream);
}

int longspec_hta_selftest_wait_timeout(void *workspace, cudaStream_t stream) {
    if (!workspace) return LONGSPEC_HTA_ERR_NULL_POINTER;
    if (!aligned16(workspace)) return LONGSPEC_HTA_ERR_MISALIGNED;
    DeviceInfo dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    return hta::launch_wait_timeout_selftest(static_cast<uint32_t *>(workspace), stream) == cudaSuccess
               ? LONGSPEC_HTA_OK : LONGSPEC_HTA_ERR_CUDA;
}

int longspec_hta_get_status(void *workspace, cudaStream_t stream) {
    if (!workspace) return LONGSPEC_HTA_ERR_NULL_POINTER;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return LONGSPEC_HTA_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess)
        return LONGSPEC_HTA_ERR_CUDA;
    if (word & hta::kStatusBadParent) return LONGSPEC_HTA_ERR_BAD_PARENT;
    if (word & hta::kStatusPrefixLenRange) return LONGSPEC_HTA_ERR_PREFIX_LEN_RANGE;
    if (word & hta::kStatusPipelineTimeout) return LONGSPEC_HTA_ERR_PIPELINE_TIMEOUT;
    if (word & hta::kStatusBadBlock) return LONGSPEC_HTA_ERR_BAD_BLOCK;
    if (word & hta::kStatusBadPath) return LONGSPEC_HTA_ERR_BAD_PATH;
    if (word & hta::kStatusInternal) return LONGSPEC_HTA_ERR_INTERNAL;
    return LONGSPEC_HTA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Verification without any device allocation by the caller.
//
// Some callers cannot allocate device memory for a workspace: a serving
// engine that reserves all device memory for its weights and KV cache at
// start-up and allows no later allocation, or a latency-critical decode
// step in which a cudaMalloc would synchronise the device.  For them the
// scratch (status word and prefix split partials) lives in this file-scope
// device array instead.  Every GPU that loads the library holds it until
// the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The array's address belongs to the context the module was loaded in:
// after a device reset, or with another context current on the same device
// (a driver-API context instead of the primary one), the module is loaded
// again, possibly elsewhere.  So the cached address is keyed on the current
// context as well as the device, and looked up again when that changes.
struct NoAllocSlot {
    CUcontext ctx;
    void *ptr;
};
NoAllocSlot g_noalloc[kMaxDevices];
std::mutex g_noalloc_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

// Device address of the static scratch in the current context
// (cudaGetSymbolAddress, a query, not an allocation).  In host code the
// array's name only stands in for it and must never reach a kernel.
int noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LONGSPEC_HTA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return LONGSPEC_HTA_ERR_UNSUPPORTED_DEVICE;
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (!get_ctx) return LONGSPEC_HTA_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return LONGSPEC_HTA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    NoAllocSlot &slot = g_noalloc[dev];
    if (!slot.ptr || !ctx || slot.ctx != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LONGSPEC_HTA_ERR_CUDA;
        // the lookup makes the device's primary context current if none was
        if (!ctx && get_ctx(&ctx) != CUDA_SUCCESS) return LONGSPEC_HTA_ERR_CUDA;
        slot.ctx = ctx;
        slot.ptr = p;
    }
    *out = slot.ptr;
    return LONGSPEC_HTA_OK;
}

// The split-KV chunking the no-allocation call uses on a GPU with `num_sms`
// SMs: the usual choice, or the largest smaller split count whose partials
// fit in the static scratch.  ok = false: not even one split fits.
Chunking noalloc_chunking(const longspec_hta_dims *dims, int num_sms, bool *ok) {
    int S = chunking_for(dims, 0, num_sms).S;
    while (S > 1 && ws_layout(dims, chunking_for(dims, S, num_sms).S).total > kNoAllocScratchBytes) --S;
    const Chunking c = chunking_for(dims, S, num_sms);
    *ok = ws_layout(dims, c.S).total <= kNoAllocScratchBytes;
    return c;
}

}  // namespace

extern "C" int longspec_hta_noalloc_chunking(const longspec_hta_dims *dims, int num_sms,
                                             int *num_splits_out, int *chunk_keys_out) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (num_sms < 1) return LONGSPEC_HTA_ERR_INVALID_OPTION;
    bool ok = false;
    const Chunking c = noalloc_chunking(dims, num_sms, &ok);
    if (!ok) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    if (num_splits_out) *num_splits_out = c.S;
    if (chunk_keys_out) *chunk_keys_out = c.chunk_tiles * hta::kKeyTile;
    return LONGSPEC_HTA_OK;
}

extern "C" int longspec_hta_verify_noalloc(const longspec_hta_dims *dims, const void *q,
                                           const void *k_prefix, const void *v_prefix,
                                           const int32_t *prefix_len, const void *k_tree,
                                           const void *v_tree, const int32_t *parent, void *out,
                                           float *lse, cudaStream_t stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    const void *ptrs[] = {q, k_prefix, v_prefix, prefix_len, k_tree, v_tree, parent, out, lse};
    for (const void *p : ptrs) {
        if (!p) return LONGSPEC_HTA_ERR_NULL_POINTER;
        if (!aligned16(p)) return LONGSPEC_HTA_ERR_MISALIGNED;
    }
    DeviceInfo di;
    if ((rc = current_device(&di))) return rc;
    // the largest split count up to the usual choice whose partials fit
    bool fits = false;
    const Chunking c = noalloc_chunking(dims, di.num_sms, &fits);
    if (!fits) return LONGSPEC_HTA_ERR_WORKSPACE_TOO_SMALL;
    const WsLayout w = ws_layout(dims, c.S);
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch))) return rc;
    uint8_t *ws = static_cast<uint8_t *>(scratch);
    // the array keeps the previous call's contents: the status word must
    // start at zero; the partials are fully written before they are read
    if (cudaMemsetAsync(ws, 0, hta::kStatusBytes, stream) != cudaSuccess) return LONGSPEC_HTA_ERR_CUDA;
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    float *o_part = reinterpret_cast<float *>(ws + w.o_off);
    float *lse_part = reinterpret_cast<float *>(ws + w.lse_off);
    const PrefixParams pp = prefix_params(dims, c, q, k_prefix, v_prefix, prefix_len, o_part, lse_part, status);
    if ((rc = run_prefix(dims, pp, LONGSPEC_HTA_PREFIX_TCGEN05, nullptr, nullptr, stream))) return rc;
    TreeMergeParams tp = tree_params(dims, hta::kTreeModeMerge, c.S, q, k_tree, v_tree, parent,
                                     prefix_len, o_part, lse_part, status);
    tp.out = static_cast<__nv_bfloat16 *>(out);
    tp.lse = lse;
    return hta::launch_tree_merge(tp, stream) == cudaSuccess ? LONGSPEC_HTA_OK : LONGSPEC_HTA_ERR_CUDA;
}
