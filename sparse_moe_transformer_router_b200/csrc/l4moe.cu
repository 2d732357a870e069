// l4moe.cu -- host side of the C ABI declared in include/l4moe.h: argument
// checks, workspace layout, TMA descriptor cache and the launch sequence
//
//   router -> permute (counts, scan, slots, work lists) -> copy of x into
//   expert order -> grouped gate/up (shared expert + routed experts; gate and
//   SwiGLU in the epilogue; + a finish kernel when split over K) -> grouped
//   down (shared and routed results as fp32 partials, un-permuted) -> finish
//   (sum, one rounding)
//
// all enqueued on the caller's stream with no host synchronisation, each
// kernel launched with programmatic stream serialisation.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "l4moe.h"
#include "finish.cuh"
#include "moe_gemm.cuh"
#include "permute.cuh"
#include "quant.cuh"
#include "route_small.cuh"
#include "router.cuh"

using namespace l4moe;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major tensor [outer, inner] with 128-byte swizzled boxes.
bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Split-K is used for batches of at most this many tokens, into at most
// kMaxSplit k-ranges (tiles too few to fill the GPU, e.g. decode).
constexpr size_t kSplitMaxTokens = 64;
constexpr int kMaxSplit = 16;
// The expert-split router (one token tile) also splits K into this many
// slices, one cluster of CTAs per 16-expert chunk.
constexpr int kRouterKSplit = 8;

struct WsLayout {
    size_t err, idx, gate, lmax, margin, inv, perm, gslot, counts, offsets, chunk, tab_gu, tab_dn, xg, hr,
        hs, x16, xsc, hq, hsc, part, logits, xin, xout;
    size_t device_total;  // everything l4moe_forward uses
    size_t total;         // plus the host-path staging slots (last)
};

size_t act_bytes(l4moe_dtype dt) { return dt == L4MOE_F32 ? 4 : 2; }
// Bytes of a row of n weights (int4: two per byte).
uint64_t w_row_bytes(l4moe_dtype dt, uint64_t n) {
    return dt == L4MOE_F32 ? 4 * n : dt == L4MOE_BF16 ? 2 * n : dt == L4MOE_INT4 ? n / 2 : n;
}
// coded weights (E4M3, int8 or int4) with per-output-column scales, widened
// to f16 in the GEMMs (the activations of these layers are f16 there)
bool coded8(l4moe_dtype dt) { return dt == L4MOE_FP8_E4M3 || dt == L4MOE_INT8 || dt == L4MOE_INT4; }

// Split-K plan of one forward of T tokens: how many k-ranges the gate/up and
// the down launches use.  Only batches of at most kSplitMaxTokens split, into
// ranges of at least 8 k-blocks.
struct SplitPlan {
    int s_gu, s_dn;
    bool fused;  // gate/up and down in one launch (small batches, see run_layer)
};

SplitPlan split_plan(const l4moe_params& p, int T, int sms, int k = 1, bool act8 = false) {
    const int d = p.d_model, F = p.expert_ffn, Fs = p.shared_ffn, E = p.num_experts;
    // K elements per k-block (one 128-byte token row; E4M3 rows in the FP8 activation mode)
    const int kblk = act8 ? 128 : (int)(128 / act_bytes(p.dtype));
    const int fb_gu_r = (F + 127) / 128, fb_gu_s = (Fs + 127) / 128, fb_dn = (d + 255) / 256;
    // Tiles are striped over the CTA pairs, so the launch lasts ceil(units /
    // pairs) tile times: take the split count that fills the last wave best
    // (fewer splits unless more fill it clearly better).
    const long long pairs = std::max(1, sms / 2);
    auto pick = [&](long long tiles, int nkb) {
        if ((size_t)T > kSplitMaxTokens || tiles <= 0) return 1;
        const int max_sp = std::min(kMaxSplit, std::max(1, nkb / 8));
        int best = 1;
        double best_fill = 0.0;
        for (int sp = 1; sp <= max_sp; ++sp) {
            const long long units = tiles * sp;
            const long long waves = (units + pairs - 1) / pairs;
            const double fill = (double)units / (double)(waves * pairs);
            if (fill > best_fill + 0.02) {
                best = sp;
                best_fill = fill;
            }
        }
        return best;
    };
    const long long eg = std::min<long long>(E, (long long)T * k);  // non-empty routed experts
    SplitPlan sp;
    const long long gu_tiles = (long long)fb_gu_s + fb_gu_r * eg;
    // On decode batches of a Maverick-shaped layer a split gate/up launch
    // (partials plus a finish kernel) was slower than the unsplit one whenever
    // at least half of the pairs had a tile (T = 1: 73 against 68 us), so
    // gate/up splits only below that.
    sp.s_gu = 2 * gu_tiles < pairs ? pick(gu_tiles, d / kblk) : 1;
    sp.s_dn = pick((long long)fb_dn * (eg + 1), std::min(F, Fs) / kblk);
    // small batches of layers whose shared operand is x run both GEMMs as one
    // launch (when gate/up needs no split); there the down units share the
    // pairs with the gate/up tiles, and units about as long as a gate/up tile
    // (a K split of about min(F, Fs) / d, ranges of at least 8 k-blocks)
    // packed best (Maverick decode, T = 1: 2 splits 0.109 ms, 4 0.113, 11
    // -- the fill-the-wave count of a down launch alone -- 0.121, 16 0.133)
    sp.fused = E > 0 && T <= kSmallMaxTokens && !coded8(p.dtype) && sp.s_gu == 1;
    if (sp.fused) {
        const int nkb = std::min(F, Fs) / kblk;
        sp.s_dn = std::max(1, std::min({kMaxSplit, std::max(1, nkb / 8),
                                        (int)((std::min(F, Fs) + d / 2) / d)}));
    }
    return sp;
}

// fp32 partial floats any forward of at most T tokens needs: split gate/up
// results, and the down's shared + routed results (times its splits).
size_t part_floats(const l4moe_params& p, int T, int sms, int k, bool act8) {
    size_t need = 0;
    auto add = [&](int t) {  // t tokens: t * k routed entries, t shared rows
        const SplitPlan sp = split_plan(p, t, sms, k, act8);
        const size_t tv = (size_t)t * k;
        if (sp.s_gu > 1)
            need = std::max<size_t>(need, (size_t)sp.s_gu * (tv * 2ull * p.expert_ffn + (size_t)t * 2ull * p.shared_ffn));
        need = std::max<size_t>(need, (size_t)sp.s_dn * (tv + t) * p.d_model);
    };
    for (int t = 1; t <= std::min<int>(T, (int)kSplitMaxTokens); ++t) add(t);
    add(std::max(T, 1));
    return need;
}

// k: selected experts per token (l4moe_set_top_k); the routed rows are the
// T * k token entries.  act8: the FP8 activation mode (E4M3 hidden rows and
// their scales).
WsLayout ws_layout(const l4moe_params& p, int T, int sms, int k, bool act8 = false) {
    WsLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 255) & ~size_t(255);
        return o;
    };
    const size_t t = (size_t)std::max(T, 1), E = (size_t)p.num_experts, es = act_bytes(p.dtype);
    const size_t tv = t * (size_t)k;
    L.err = take(256);  // device error word, the routing kernels' ticket, the fused GEMM's two
                        // tile counters (zeroed once; each user leaves them at zero)
    L.idx = take(4 * tv);
    L.gate = take(4 * tv);
    L.lmax = take(4 * tv);
    L.margin = take(4 * t);
    L.inv = take(4 * tv);
    L.perm = take(4 * tv);
    L.gslot = take(4 * tv);
    L.counts = take(4 * E);
    L.offsets = take(4 * (E + 1));
    L.chunk = take(4 * router_max_chunks(tv) * E);  // dispatch chunk bases (either dispatch)
    L.tab_gu = take(sizeof(GroupTable));
    L.tab_dn = take(sizeof(GroupTable));
    L.xg = take(tv * p.d_model * es);
    L.hr = take(tv * p.expert_ffn * es);
    L.hs = take(t * p.shared_ffn * es);
    // 8-bit weight layers: x in f16, token order (the shared expert's operand)
    L.x16 = take(coded8(p.dtype) ? t * p.d_model * 2 : 0);
    L.xsc = take(coded8(p.dtype) ? 4 * t : 0);  // and each token row's scale
    // FP8 activation mode: the hidden rows' E4M3 codes (routed [T k][F], then
    // shared [T][Fs]) and their row scales ([T k] then [T])
    L.hq = take(act8 ? tv * p.expert_ffn + t * p.shared_ffn : 0);
    L.hsc = take(act8 ? 4 * (tv + t) : 0);
    L.part = take(sizeof(float) * part_floats(p, (int)t, sms, k, act8));
    // expert-split router logits [min(T, 128)][E]; for batches the one-launch
    // routing takes, its partial logits [slices][T][E]
    const size_t small_part = (size_t)((p.d_model + kSmallSliceK - 1) / kSmallSliceK) *
                              std::min<size_t>(t, kSmallMaxTokens) * E;
    L.logits = take(sizeof(float) * std::max(std::min<size_t>(t, 128) * E, small_part));
    L.device_total = off;
    L.xin = take(2 * t * p.d_model * es);   // host path: two input staging slots
    L.xout = take(2 * t * p.d_model * es);  // and two output staging slots
    L.total = off;
    return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

struct l4moe_handle {
    l4moe_params p{};
    int device = -1;
    int sms = 0;
    uint8_t* ws = nullptr;
    size_t ws_bytes = 0;
    int ws_tokens = 0;
    int top_k = 1;  // selected experts per token (l4moe_set_top_k)
    bool act8 = false;  // FP8 activation mode (l4moe_set_act_fp8)
    bool ws_owned = false;
    const float* bias = nullptr;
    std::vector<const float*> s_gu, s_dn;
    const float* ss_gu = nullptr;
    const float* ss_dn = nullptr;
    const float** d_scales = nullptr;  // device [2][E+1] scale pointers (gate/up, down)
    bool scales_dirty = false;
    // host copy of that table, the source of every upload: sized once at
    // creation and rewritten in place by l4moe_set_weight_scales, so its
    // address stays fixed for the handle's life (a copy recorded under stream
    // capture reads it again at every replay)
    std::vector<const float*> scale_tab;
    // TMA descriptors of the weights, keyed by pointer value
    std::vector<const void*> key_gu, key_dn;
    const void* key_sgu = nullptr;
    const void* key_sdn = nullptr;
    std::vector<CUtensorMap> h_maps;  // [2][E+1]: gate/up set then down set; capacity
                                      // reserved at creation, so its address is fixed
    std::vector<const void*> hkey_gu, hkey_dn;  // weights h_maps was encoded for
    const void* hkey_sgu = nullptr;
    const void* hkey_sdn = nullptr;
    CUtensorMap* d_maps = nullptr;
    uint64_t launches = 0;
    std::string err;
    int last_T = 0;
    l4moe_plan last_plan{};  // launch plan of the last forward
    // host path (l4moe_forward_host): copy streams and per-slot events so
    // consecutive calls overlap their copies with each other's compute
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_h2d[2] = {}, ev_comp[2] = {}, ev_d2h[2] = {};
    bool slot_used[2] = {false, false};
    int host_slot = 0;
    // per-kernel event timing (l4moe_set_timing): bit i times kernel slot i
    unsigned timing = 0;
    std::vector<cudaEvent_t> ev_pool;             // recycled events
    std::vector<std::pair<int, std::pair<cudaEvent_t, cudaEvent_t>>> ev_pending;
};

namespace {

thread_local std::string g_create_error;

l4moe_status fail(l4moe_handle* h, l4moe_status s, const std::string& msg) {
    if (h) h->err = msg;
    else g_create_error = msg;
    return s;
}

l4moe_status cuda_fail(l4moe_handle* h, cudaError_t e, const char* what) {
    return fail(h, L4MOE_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

cudaEvent_t take_event(l4moe_handle* h) {
    if (!h->ev_pool.empty()) {
        cudaEvent_t e = h->ev_pool.back();
        h->ev_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Every kernel goes out with programmatic stream serialisation: it may begin
// launching while the previous kernel of the stream finishes, and waits for
// it (pdl_enter) before touching memory, which hides the launch gaps of the
// short kernels of a small batch.  Launch errors are left for
// cudaGetLastError, like a <<<>>> launch.
// cluster_z > 0 also launches the grid as clusters of (1, 1, cluster_z).
template <typename... KArgs, typename... Args>
void launch_kc(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
               unsigned cluster_z, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 1;
    if (cluster_z > 0) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = 1;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = cluster_z;
        cfg.numAttrs = 2;
    }
    cfg.attrs = attr;
    cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
void launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
              Args&&... args) {
    launch_kc(kernel, grid, block, smem, st, 0u, std::forward<Args>(args)...);
}

// Event pair around one launch when timing is enabled.
struct LaunchTimer {
    l4moe_handle* h;
    int slot;
    cudaStream_t st;
    cudaEvent_t a = nullptr, b = nullptr;
    LaunchTimer(l4moe_handle* h_, int slot_, cudaStream_t st_) : h(h_), slot(slot_), st(st_) {
        if ((h->timing >> slot_ & 1u) && (a = take_event(h)) != nullptr) cudaEventRecord(a, st);
    }
    void stop() {
        if (a && (b = take_event(h)) != nullptr) {
            cudaEventRecord(b, st);
            h->ev_pending.push_back({slot, {a, b}});
        }
    }
};

l4moe_status ensure_workspace(l4moe_handle* h, int T) {
    if (h->ws && T <= h->ws_tokens) return L4MOE_OK;
    if (h->ws && !h->ws_owned)
        return fail(h, L4MOE_ERR_WORKSPACE, "caller workspace is sized for fewer tokens than T");
    if (h->ws_owned && h->ws) {
        cudaFree(h->ws);  // implicit device sync; only when T grows
        h->ws = nullptr;
    }
    const int cap = std::max(T, 256);
    const WsLayout L = ws_layout(h->p, cap, h->sms, h->top_k, h->act8);
    void* p = nullptr;
    cudaError_t e = cudaMalloc(&p, L.total);
    if (e != cudaSuccess) return cuda_fail(h, e, "workspace cudaMalloc");
    e = cudaMemset(p, 0, 256);
    if (e != cudaSuccess) return cuda_fail(h, e, "workspace cudaMemset");
    h->ws = static_cast<uint8_t*>(p);
    h->ws_bytes = L.total;
    h->ws_tokens = cap;
    h->ws_owned = true;
    return L4MOE_OK;
}

// Encode the weight descriptors on the host (h->h_maps) unless they already
// describe these pointers.
l4moe_status encode_weight_maps(l4moe_handle* h, const void* const* Wgu, const void* const* Wdn,
                                const void* Wsgu, const void* Wsdn) {
    const int E = h->p.num_experts;
    bool same = !h->h_maps.empty() && h->hkey_sgu == Wsgu && h->hkey_sdn == Wsdn;
    for (int e = 0; same && e < E; ++e) same = h->hkey_gu[e] == Wgu[e] && h->hkey_dn[e] == Wdn[e];
    if (same) return L4MOE_OK;
    const int d = h->p.d_model, F = h->p.expert_ffn, Fs = h->p.shared_ffn;
    const l4moe_dtype wdt = h->p.dtype;
    CUtensorMapDataType dt = wdt == L4MOE_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                             : wdt == L4MOE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const bool act8 = h->act8;               // E4M3 codes read raw by the MMA
    const bool fp8 = coded8(wdt) && !act8;  // codes widened in shared memory
    const uint32_t bk = wdt == L4MOE_F32 ? 32 : act8 ? 128 : 64;  // K rows per box
    // box width in elements of the map: one 128-byte swizzled slab of
    // features; coded weights are staged raw (64-feature boxes, unswizzled;
    // int4 maps count bytes, 32 of them per 64 features) and widened in
    // shared memory; in the FP8 activation mode the codes land as the MMA
    // reads them: 64-feature slabs in the 64-byte swizzle
    const uint32_t bw = wdt == L4MOE_INT4 ? 32u : (fp8 || act8) ? 64u : (uint32_t)(128 / w_row_bytes(wdt, 1));
    // MN-major 32-bit operands need the 32-byte swizzle unit
    const CUtensorMapSwizzle swz = act8 ? CU_TENSOR_MAP_SWIZZLE_64B
                                   : fp8 ? CU_TENSOR_MAP_SWIZZLE_NONE
                                   : h->p.dtype == L4MOE_F32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                                                             : CU_TENSOR_MAP_SWIZZLE_128B;
    h->h_maps.assign(2 * (E + 1), CUtensorMap{});
    h->hkey_gu.clear();
    for (int e = 0; e <= E; ++e) {
        const bool sh = (e == E);
        const void* gu = sh ? Wsgu : Wgu[e];
        const void* dn = sh ? Wsdn : Wdn[e];
        const int f = sh ? Fs : F;
        // map elements per row: features, or bytes for int4
        const uint64_t gu_w = wdt == L4MOE_INT4 ? (uint64_t)f : 2ull * f;
        const uint64_t dn_w = wdt == L4MOE_INT4 ? (uint64_t)d / 2 : (uint64_t)d;
        if (!encode_2d(&h->h_maps[e], dt, gu, gu_w, (uint64_t)d, w_row_bytes(wdt, 2ull * f), bw, bk, swz) ||
            !encode_2d(&h->h_maps[E + 1 + e], dt, dn, dn_w, (uint64_t)f, w_row_bytes(wdt, (uint64_t)d), bw,
                       bk, swz)) {
            h->h_maps.clear();
            return fail(h, L4MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for a weight");
        }
    }
    h->hkey_gu.assign(Wgu, Wgu + E);
    h->hkey_dn.assign(Wdn, Wdn + E);
    h->hkey_sgu = Wsgu;
    h->hkey_sdn = Wsdn;
    return L4MOE_OK;
}

// (Re)build and upload the weight descriptors when any weight pointer changed.
l4moe_status ensure_weight_maps(l4moe_handle* h, const void* const* Wgu, const void* const* Wdn,
                                const void* Wsgu, const void* Wsdn, cudaStream_t st) {
    const int E = h->p.num_experts;
    bool same = h->d_maps && h->key_sgu == Wsgu && h->key_sdn == Wsdn;
    for (int e = 0; same && e < E; ++e) same = h->key_gu[e] == Wgu[e] && h->key_dn[e] == Wdn[e];
    if (same) return L4MOE_OK;
    l4moe_status s = encode_weight_maps(h, Wgu, Wdn, Wsgu, Wsdn);
    if (s != L4MOE_OK) return s;
    if (!h->d_maps) {
        cudaError_t e = cudaMalloc(&h->d_maps, sizeof(CUtensorMap) * 2 * (E + 1));
        if (e != cudaSuccess) return cuda_fail(h, e, "descriptor cudaMalloc");
    }
    // pageable source: returns once the bytes are staged, so h_maps may change later
    cudaError_t e = cudaMemcpyAsync(h->d_maps, h->h_maps.data(), sizeof(CUtensorMap) * 2 * (E + 1),
                                    cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "descriptor upload");
    h->key_gu.assign(Wgu, Wgu + E);
    h->key_dn.assign(Wdn, Wdn + E);
    h->key_sgu = Wsgu;
    h->key_sdn = Wsdn;
    return L4MOE_OK;
}

template <typename K>
void set_smem_attr(K kernel, size_t bytes) {
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Raise a kernel's dynamic shared-memory limit once per device: the
// attribute belongs to the kernel's instance in each device's context, so a
// process that runs layers on several GPUs sets it on each.  `done` holds
// one bit per device index (devices 64 and up set it on every call).
template <typename K>
void ensure_smem_attr(std::atomic<uint64_t>& done, K kernel, size_t bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        set_smem_attr(kernel, bytes);
        return;
    }
    const uint64_t bit = 1ull << dev;
    if (done.load(std::memory_order_acquire) & bit) return;
    set_smem_attr(kernel, bytes);
    done.fetch_or(bit, std::memory_order_acq_rel);
}

template <typename ET, int NT, int TPT, int NG>
void launch_router_t(const void* x, const void* Wr, const float* bias, int T, int d, int E,
                     int32_t* idx, float* gate, float* lmax, float* margin, int k, cudaStream_t st) {
    constexpr size_t smem = router_smem_bytes<NT, TPT, NG>();
    static std::atomic<uint64_t> attr_done{0};
    ensure_smem_attr(attr_done, router_kernel<ET, NT, TPT, NG>, smem);
    const int TT = NT / TPT;
    const int wr_vec = (E % Vec16<ET>::N) == 0 ? 1 : 0;
    launch_k(router_kernel<ET, NT, TPT, NG>, dim3((T + TT - 1) / TT), dim3(NT), smem, st,
             static_cast<const ET*>(x), static_cast<const ET*>(Wr), bias, T, d, E, wr_vec, idx, gate,
             lmax, margin, k);
}

template <typename ET>
void launch_router(const void* x, const void* Wr, const float* bias, int T, int d, int E,
                   int32_t* idx, float* gate, float* lmax, float* margin, int k, cudaStream_t st) {
    const int EG = (E + 3) / 4;
    if (EG <= 1) launch_router_t<ET, 128, 1, 1>(x, Wr, bias, T, d, E, idx, gate, lmax, margin, k, st);
    else if (EG <= 2) launch_router_t<ET, 128, 2, 1>(x, Wr, bias, T, d, E, idx, gate, lmax, margin, k, st);
    else if (EG <= 4) launch_router_t<ET, 128, 4, 1>(x, Wr, bias, T, d, E, idx, gate, lmax, margin, k, st);
    else if (EG <= 8) launch_router_t<ET, 128, 8, 1>(x, Wr, bias, T, d, E, idx, gate, lmax, margin, k, st);
    else if (EG <= 16) launch_router_t<ET, 256, 8, 2>(x, Wr, bias, T, d, E, idx, gate, lmax, margin, k, st);
    else if (EG <= 32) launch_router_t<ET, 256, 8, 4>(x, Wr, bias, T, d, E, idx, gate, lmax, margin, k, st);
    else launch_router_t<ET, 256, 8, 8>(x, Wr, bias, T, d, E, idx, gate, lmax, margin, k, st);
}

// bm / a: the GEMM (a fused launch's gate/up); bm2 / a2: a fused launch's down
template <int MODE, typename ET, int WQ, bool SMALLN>
void launch_gemm_cfg(int grid, const BMaps& bm, const GemmArgs& a, const BMaps& bm2, const GemmArgs& a2,
                     cudaStream_t st) {
    using Cfg = GemmCfg<MODE, ET, WQ, SMALLN>;
    static std::atomic<uint64_t> attr_done{0};
    ensure_smem_attr(attr_done, moe_gemm_kernel<MODE, ET, WQ, SMALLN>, Cfg::SMEM_BYTES);
    launch_k(moe_gemm_kernel<MODE, ET, WQ, SMALLN>, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM_BYTES, st, bm, a,
             bm2, a2);
}

// small: every group of the launch has at most 64 rows (the small-batch
// configuration with the deeper weight ring)
template <int MODE, typename ET, int WQ>
void launch_gemm_pair(int grid, const BMaps& bm, const GemmArgs& a, const BMaps& bm2, const GemmArgs& a2,
                      cudaStream_t st, bool small) {
    if (small) launch_gemm_cfg<MODE, ET, WQ, true>(grid, bm, a, bm2, a2, st);
    else launch_gemm_cfg<MODE, ET, WQ, false>(grid, bm, a, bm2, a2, st);
}

template <int MODE, typename ET, int WQ>
void launch_gemm(int grid, const BMaps& bm, const GemmArgs& a, cudaStream_t st, bool small) {
    launch_gemm_pair<MODE, ET, WQ>(grid, bm, a, bm, a, st, small);
}

// The launch sequence of one forward.  w / ws_tokens: the workspace and the
// token count its layout was made for; maps: device array of the 2(E+1)
// weight descriptors.
// WQ: the weights' storage (kWqNone: the layer's type; kWqE4M3 / kWqInt8 /
// kWqInt4: codes with per-column scales, widened to f16 in the GEMMs;
// kWqAct8: E4M3 codes multiplied raw with E4M3 token rows, the FP8
// activation mode).
template <typename ET, int WQ = kWqNone>
l4moe_status run_layer(l4moe_handle* h, int T, const void* x, const void* Wr, const void* Wsgu,
                       const void* Wsdn, void* out, cudaStream_t st, uint8_t* w, int ws_tokens,
                       const CUtensorMap* maps, const float* const* scales = nullptr) {
    constexpr bool FP8W = WQ != kWqNone;  // coded weights with per-column scales
    constexpr bool ACT8 = WQ == kWqAct8;  // and E4M3 token rows (FP8 activation mode)
    const l4moe_params& p = h->p;
    const int d = p.d_model, F = p.expert_ffn, Fs = p.shared_ffn, E = p.num_experts;
    const WsLayout L = ws_layout(p, ws_tokens, h->sms, h->top_k, h->act8);
    unsigned* err = reinterpret_cast<unsigned*>(w + L.err);
    int32_t* idx = reinterpret_cast<int32_t*>(w + L.idx);
    float* gate = reinterpret_cast<float*>(w + L.gate);
    float* lmax = reinterpret_cast<float*>(w + L.lmax);
    float* margin = reinterpret_cast<float*>(w + L.margin);
    int32_t* inv = reinterpret_cast<int32_t*>(w + L.inv);
    int32_t* perm = reinterpret_cast<int32_t*>(w + L.perm);
    float* gslot = reinterpret_cast<float*>(w + L.gslot);
    int32_t* counts = reinterpret_cast<int32_t*>(w + L.counts);
    int32_t* offsets = reinterpret_cast<int32_t*>(w + L.offsets);
    GroupTable* tab_gu = reinterpret_cast<GroupTable*>(w + L.tab_gu);
    GroupTable* tab_dn = reinterpret_cast<GroupTable*>(w + L.tab_dn);
    // the hidden rows' type: the layer's, or f16 for widened coded weights
    // (kind::f16 wants both operands of one type); the token operand's type:
    // the same, or E4M3 codes in the FP8 activation mode (hidden rows then
    // stay bf16 until their own quantisation)
    using HT = typename GemmAct<ET, FP8W && !ACT8>::type;
    using GT = typename std::conditional<ACT8, uint8_t, HT>::type;
    GT* xg = reinterpret_cast<GT*>(w + L.xg);
    HT* hr = reinterpret_cast<HT*>(w + L.hr);
    HT* hs = reinterpret_cast<HT*>(w + L.hs);
    GT* x16 = reinterpret_cast<GT*>(w + L.x16);
    float* tokscale = FP8W ? reinterpret_cast<float*>(w + L.xsc) : nullptr;
    // FP8 activation mode: hidden-row codes and scales (routed, then shared)
    uint8_t* hq_r = ACT8 ? w + L.hq : nullptr;
    float* hsc_r = ACT8 ? reinterpret_cast<float*>(w + L.hsc) : nullptr;

    // per-call activation descriptors (K-major rows of 128 B): the router's
    // x (64-row boxes) and the GEMMs' token operands (full- and small-tile
    // boxes: gate/up reads x in expert order and x, down reads H_r and H_s)
    auto tmap_type = [](size_t bytes, bool f16) {
        return bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
               : bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
               : f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    };
    const CUtensorMapDataType adt = tmap_type(sizeof(ET), false);
    const CUtensorMapDataType gdt = tmap_type(sizeof(GT), FP8W);  // gate/up token operand
    const CUtensorMapDataType ddt = ACT8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : gdt;  // down's: hidden rows
    const size_t dsz = ACT8 ? 1 : sizeof(HT);
    using GCfg = GemmCfg<MODE_GATEUP, ET, WQ>;
    constexpr uint32_t rb = GCfg::B_BOX_ROWS, rs = GCfg::B_SMALL_ROWS;
    CUtensorMap m_x;
    BMaps bm_gu, bm_dn;
    // rows: T token rows (x, the shared hidden rows), or T * k entries for
    // the routed rows (x in expert order, the routed hidden rows)
    const int k = h->top_k;
    const int Tv = T * k;
    // K-major rows, boxes of 128 bytes of K by `rows` rows; esz: element bytes
    auto act_n = [&](CUtensorMap* m, CUtensorMapDataType dt, const void* base, int width, int nrows,
                     uint32_t rows, size_t esz) {
        return encode_2d(m, dt, base, (uint64_t)width, (uint64_t)nrows, (uint64_t)width * esz,
                         (uint32_t)(128 / esz), rows);
    };
    auto act = [&](CUtensorMap* m, CUtensorMapDataType dt, const void* base, int width, uint32_t rows,
                   size_t esz) { return act_n(m, dt, base, width, T, rows, esz); };
    auto act_r = [&](CUtensorMap* m, CUtensorMapDataType dt, const void* base, int width, uint32_t rows,
                     size_t esz) { return act_n(m, dt, base, width, Tv, rows, esz); };
    const void* xs = FP8W ? (const void*)x16 : x;  // the shared expert's operand
    // the down's token operand: the hidden rows, or their codes in the FP8
    // activation mode (routed [Tv][F] then shared [T][Fs])
    const void* hdr = ACT8 ? (const void*)hq_r : (const void*)hr;
    const void* hds = ACT8 ? (const void*)(hq_r + (size_t)Tv * F) : (const void*)hs;
    // without experts (F may be 0) the routed hidden descriptors are never
    // read: give them the shared hidden rows to describe
    const void* hrm = F > 0 ? hdr : hds;
    const int Fr = F > 0 ? F : Fs;
    const size_t gsz = sizeof(GT);
    if (!act(&m_x, adt, x, d, 64, sizeof(ET)) || !act_r(&bm_gu.routed, gdt, xg, d, rb, gsz) ||
        !act_r(&bm_gu.routed_small, gdt, xg, d, rs, gsz) || !act(&bm_gu.shared, gdt, xs, d, rb, gsz) ||
        !act(&bm_gu.shared_small, gdt, xs, d, rs, gsz) || !act_r(&bm_dn.routed, ddt, hrm, Fr, rb, dsz) ||
        !act_r(&bm_dn.routed_small, ddt, hrm, Fr, rs, dsz) || !act(&bm_dn.shared, ddt, hds, Fs, rb, dsz) ||
        !act(&bm_dn.shared_small, ddt, hds, Fs, rs, dsz))
        return fail(h, L4MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for an activation");

    cudaError_t e;
#define L4MOE_CHECK_LAUNCH(what)                                  \
    do {                                                          \
        ++h->launches;                                            \
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(h, e, what); \
    } while (0)

    // feature blocks per pair tile: 128 features for gate/up, 256 for down
    const int fpg = pair_features<MODE_GATEUP>(), fpd = pair_features<MODE_DOWN>();
    const int fb_gu_r = (F + fpg - 1) / fpg;
    const int fb_gu_s = (Fs + fpg - 1) / fpg;
    const int fb_dn = (d + fpd - 1) / fpd;
    // split-K k-ranges when a small batch leaves too few tiles
    const SplitPlan plan = split_plan(p, T, h->sms, h->top_k, ACT8);
    const int s_gu = plan.s_gu, s_dn = plan.s_dn;
    if (E > 0 && T <= kSmallMaxTokens) {
        // a few tokens: router, top-k, permutation and row copy in one launch
        const int slices = (d + kSmallSliceK - 1) / kSmallSliceK;
        float* part_logits = reinterpret_cast<float*>(w + L.logits);
        unsigned* ticket = err + 1;  // zero between launches (each last CTA resets it)
        static std::atomic<uint64_t> attr_done{0};
        ensure_smem_attr(attr_done, route_small_kernel<ET, GT>, route_small_smem_bytes<ET>(kSmallMaxTokens, 256));
        LaunchTimer t_router(h, 0, st);
        launch_k(route_small_kernel<ET, GT>, dim3(slices), dim3(kSmallThreads), route_small_smem_bytes<ET>(T, E), st,
                 static_cast<const ET*>(x), static_cast<const ET*>(Wr), (const float*)h->bias, T, d, E, k,
                 part_logits, ticket, idx, gate, lmax, margin, counts, offsets, perm, inv, gslot, tab_gu, tab_dn,
                 fb_gu_r * s_gu, fb_gu_s * s_gu, fb_dn * s_dn, xg, FP8W ? x16 : (GT*)nullptr, tokscale);
        t_router.stop();
        L4MOE_CHECK_LAUNCH("small-batch routing launch");
    } else if (E > 0) {
        LaunchTimer t_router(h, 0, st);
        // one token tile and many experts: split the router over 16-expert chunks
        const bool split_router = sizeof(ET) == 2 && E % 16 == 0 && E >= 32 && T <= 128;
        float* logits = split_router ? reinterpret_cast<float*>(w + L.logits) : nullptr;
        int32_t* chunk_base = logits ? nullptr : reinterpret_cast<int32_t*>(w + L.chunk);
        // the tensor-core top-1 router finishes the dispatch itself (a chunk per CTA)
        const bool router_dispatch = sizeof(ET) == 2 && E % 8 == 0 && !split_router && k == 1 &&
                                     router_max_chunks(T) <= (size_t)router_stage_cap(E);
        int router_slices = 1;  // K slices of the tensor-core router launch
        if (sizeof(ET) == 2 && E % 8 == 0) {
            // tensor-core router: W_router [d, E] as the MN-major operand
            CUtensorMap m_wr;
            if (!encode_2d(&m_wr, adt, Wr, (uint64_t)E, (uint64_t)d, (uint64_t)E * sizeof(ET), 64, 64))
                return fail(h, L4MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the router weight");
            static std::atomic<uint64_t> attr_done{0};
            ensure_smem_attr(attr_done, router_mma_kernel, rmma::SMEM_BYTES);
            const int n_chunk = split_router ? 16 : E;
            const int tiles = (T + 127) / 128;
            // stages sized for this launch's experts; two CTAs share an SM
            // when that leaves each at most half of its shared memory
            const int nst = rmma::stages(n_chunk);
            const size_t rsmem = rmma::smem_bytes(n_chunk, nst);
            const int per_sm = rsmem <= 112 * 1024 ? 2 : 1;
            int kslices;
            if (split_router) {
                kslices = std::min(kRouterKSplit, std::max(1, d / 256));
            } else {
                // few token tiles: K slices per tile (a cluster of at most 8,
                // at most the resident CTAs' worth), reduced inside the cluster
                kslices = std::max(1, std::min({4 * per_sm, per_sm * h->sms / tiles, d / 256}));
            }
            while (kslices & (kslices - 1)) kslices &= kslices - 1;  // a power of two: it divides the tile
            router_slices = kslices;
            RouterDispatch dsp{};
            if (router_dispatch) {
                dsp.chunk_base = chunk_base;
                dsp.counts = counts;
                dsp.offsets = offsets;
                dsp.inv = inv;
                dsp.tab_gu = tab_gu;
                dsp.tab_dn = tab_dn;
                dsp.ticket = err + 1;  // zero between launches (the last CTA resets it)
                dsp.fb_gu_routed = fb_gu_r * s_gu;
                dsp.fb_gu_shared = fb_gu_s * s_gu;
                dsp.fb_down = fb_dn * s_dn;
            }
            launch_kc(router_mma_kernel, dim3(tiles, E / n_chunk, kslices), dim3(128), rsmem, st,
                      kslices == 1 ? 0u : (unsigned)kslices, m_x, m_wr, (const float*)h->bias,
                      T, d, E, n_chunk, logits, idx, gate, lmax, margin, err, k, nst, dsp);
        } else {
            launch_router<ET>(x, Wr, h->bias, T, d, E, idx, gate, lmax, margin, k, st);
        }
        t_router.stop();
        L4MOE_CHECK_LAUNCH("router launch");

        // dispatch_kernel: wcnt[32][E] (also the staging of its last CTA's
        // scan, which needs a row per chunk), tot[E], soff[E + 1]
        const size_t dchunks = (Tv + kDispatchChunk - 1) / kDispatchChunk;
        const size_t psmem = sizeof(int) * (std::max<size_t>(32 * (size_t)E, dchunks) + 2 * (size_t)E + 1);
        if (!router_dispatch) {
            LaunchTimer t_perm(h, 1, st);
            if (logits) {
                // the arg-max of the split logits and the whole permutation in one CTA
                launch_k(permute_kernel, dim3(1), dim3(1024), psmem, st, (const float*)logits,
                         gate, lmax, margin, idx, T, k, E, fb_gu_r * s_gu, fb_gu_s * s_gu, fb_dn * s_dn, counts,
                         offsets, perm, inv, tab_gu, tab_dn, err);
            } else {
                launch_k(dispatch_kernel, dim3((Tv + kDispatchChunk - 1) / kDispatchChunk), dim3(kDispatchChunk),
                         psmem, st, (const int32_t*)idx, T, k, E, fb_gu_r * s_gu, fb_gu_s * s_gu, fb_dn * s_dn,
                         chunk_base, counts, offsets, inv, tab_gu, tab_dn, err + 1, err);
            }
            t_perm.stop();
            L4MOE_CHECK_LAUNCH("permute launch");
        }
        // entries per dispatch chunk: the router's tokens per CTA, or dispatch_kernel's
        const int chunk = router_dispatch ? router_tokens_per_cta(router_slices) : kDispatchChunk;

        const int sc_blocks = std::min((Tv + 7) / 8, h->sms * 8);
        LaunchTimer t_rows(h, 2, st);
        launch_k(permute_rows_kernel<ET, GT>, dim3(sc_blocks), dim3(256), 0, st, static_cast<const ET*>(x),
                 (const float*)gate, inv, T, k, d, xg, gslot, FP8W ? x16 : (GT*)nullptr, (const int32_t*)idx,
                 (const int32_t*)chunk_base, chunk, E, perm, tokscale);
        t_rows.stop();
        L4MOE_CHECK_LAUNCH("row permutation launch");
    } else {
        // no experts (a dense feed-forward layer): the shared SwiGLU over the
        // tokens in order; the work lists hold that one group
        LaunchTimer t_perm(h, 1, st);
        launch_k(dense_table_kernel, dim3(1), dim3(32), 0, st, tab_gu, tab_dn, T, fb_gu_s * s_gu, fb_dn * s_dn);
        t_perm.stop();
        L4MOE_CHECK_LAUNCH("work list launch");
        if (FP8W) {  // the f16 copy of x the contractions of 8-bit weight layers read
            const int sc_blocks = std::min((T + 7) / 8, h->sms * 8);
            LaunchTimer t_rows(h, 2, st);
            launch_k(permute_rows_kernel<ET, GT>, dim3(sc_blocks), dim3(256), 0, st, static_cast<const ET*>(x),
                     (const float*)nullptr, (int32_t*)nullptr, T, 1, d, x16, (float*)nullptr, (GT*)nullptr,
                     (const int32_t*)nullptr, (const int32_t*)nullptr, 1, 0, (int32_t*)nullptr, tokscale);
            t_rows.stop();
            L4MOE_CHECK_LAUNCH("row conversion launch");
        }
    }

    const int tb = (T + kTokTile - 1) / kTokTile;     // shared token tiles
    const int tbv = (Tv + kTokTile - 1) / kTokTile;   // routed entry tiles (bound)
    // CTA pairs: two CTAs (one cluster) per tile, at most one pair per two SMs
    auto grid_for = [&](long long tiles) {
        return 2 * (int)std::max(1LL, std::min<long long>(h->sms / 2, tiles));
    };

    GemmArgs gu{};
    gu.table = tab_gu;
    gu.a_maps = maps;
    gu.num_experts = E;
    gu.k_routed = d;
    gu.k_shared = d;
    gu.m_routed = F;
    gu.m_shared = Fs;
    gu.up_routed = F;
    gu.up_shared = Fs;
    gu.out_routed = hr;          // routed hidden rows in slot order
    gu.ld_routed = F;
    gu.out_shared = hs;          // shared hidden rows, also stored in slot order
    gu.ld_shared = Fs;
    gu.rowmap_routed = nullptr;
    gu.rowmap_shared = nullptr;  // shared hidden rows in token order
    gu.colscale_routed = gslot;      // sigmoid gate of each routed slot (times its row scale)
    gu.colscale_shared = tokscale;   // 8-bit weights: each token row's scale, else null
    gu.wscale = FP8W ? scales : nullptr;
    float* part = reinterpret_cast<float*>(w + L.part);
    gu.ksplit = s_gu;
    gu.partial_out = s_gu > 1 ? 1 : 0;
    gu.part_routed = part;
    gu.ld_part_routed = 2LL * F;
    gu.part_stride_routed = (long long)Tv * 2 * F;
    gu.part_shared = part + (size_t)s_gu * Tv * 2 * F;
    gu.ld_part_shared = 2LL * Fs;
    gu.part_stride_shared = (long long)T * 2 * Fs;
    gu.err = err;
    // after the one-launch routing of a small batch, the shared expert's tiles
    // (operand x itself, which the routing does not write) go first in the
    // work list and may run while the routing finishes: the GEMM waits for it
    // only at its first routed tile (8- and 4-bit weight layers read the f16
    // copy of x that the routing writes, so they wait at entry)
    const bool early = E > 0 && T <= kSmallMaxTokens && !FP8W;
    gu.early_tiles = early ? fb_gu_s * s_gu * tb : 0;
    gu.early_rows = T;
    // no group can have more than 64 rows: the small-batch GEMM configuration
    const bool small_tiles = T <= 2 * GCfg::B_SMALL_ROWS && Tv <= 2 * GCfg::B_SMALL_ROWS;

    GemmArgs dn{};
    dn.table = tab_dn;
    dn.a_maps = maps + (E + 1);
    dn.num_experts = E;
    dn.k_routed = F;
    dn.k_shared = Fs;
    dn.m_routed = d;
    dn.m_shared = d;
    dn.out_routed = out;
    dn.ld_routed = d;
    dn.out_shared = out;
    dn.ld_shared = d;
    dn.rowmap_routed = perm;     // slot -> token: un-permute on store
    dn.rowmap_shared = nullptr;  // shared rows are tokens
    dn.colscale_routed = hsc_r;                       // FP8 activation mode: hidden row scales
    dn.colscale_shared = ACT8 ? hsc_r + Tv : nullptr;
    dn.wscale = FP8W ? scales + (E + 1) : nullptr;
    dn.ksplit = s_dn;
    dn.partial_out = 1;
    // partial slots: [0, s_dn) routed, [s_dn, 2 s_dn) shared
    dn.part_routed = part;
    dn.ld_part_routed = d;
    dn.part_stride_routed = (long long)Tv * d;  // routed rows: the T * k entries
    dn.part_shared = part + (size_t)s_dn * Tv * d;
    dn.ld_part_shared = d;
    dn.part_stride_shared = (long long)T * d;
    dn.err = err;
    // A small batch whose gate/up starts early and needs no split-K finish
    // runs both contractions as one launch: its pairs take the gate/up tiles
    // and then the down tiles, each down tile waiting (on device counters of
    // finished gate/up tiles) only for the hidden rows of its own class, so
    // the pairs that finish their gate/up tiles stream down weights while the
    // others still stream gate/up weights
    const bool fused = plan.fused;
    unsigned* done = fused ? err + 2 : nullptr;  // zero here; the down finish resets them
    gu.done = done;
    dn.done = done;
    h->last_plan.split_gate_up = s_gu;
    h->last_plan.split_down = s_dn;
    h->last_plan.early_shared = early ? 1 : 0;
    h->last_plan.fused = fused ? 1 : 0;
    h->last_plan.small_tiles = small_tiles ? 1 : 0;
    h->last_plan.small_routing = (E > 0 && T <= kSmallMaxTokens) ? 1 : 0;
    const long long gu_units = s_gu * ((long long)fb_gu_s * tb + (long long)fb_gu_r * (tbv + std::min(E, Tv)));
    const long long dn_units = s_dn * (long long)fb_dn * (tb + tbv + std::min(E, Tv));
    if (fused) {
        LaunchTimer t_gu(h, 3, st);
        launch_gemm_pair<MODE_FUSED, ET, WQ>(grid_for(gu_units + dn_units), bm_gu, gu, bm_dn, dn, st, small_tiles);
        t_gu.stop();
        L4MOE_CHECK_LAUNCH("fused gate/up and down launch");
    } else {
        LaunchTimer t_gu(h, 3, st);
        launch_gemm<MODE_GATEUP, ET, WQ>(grid_for(gu_units), bm_gu, gu, st, small_tiles);
        if (s_gu > 1) {
            const long long n = (long long)Tv * F + (long long)T * Fs;
            launch_k(gateup_finish_kernel<HT>, dim3((int)std::min<long long>((n + 255) / 256, 4LL * h->sms)),
                     dim3(256), 0, st, (const float*)gu.part_routed, gu.ld_part_routed, gu.part_stride_routed,
                     (const float*)gu.part_shared, gu.ld_part_shared, gu.part_stride_shared, s_gu, Tv, T, F, Fs,
                     (const float*)gslot, (const float*)tokscale, hr, hs, err);
            ++h->launches;
        }
        t_gu.stop();
        L4MOE_CHECK_LAUNCH("gate/up launch");
        if constexpr (ACT8) {
            // the hidden rows' E4M3 codes and row scales, one CTA per row at a time
            const int Tr = E > 0 ? Tv : 0;
            const int rows = Tr + T;
            LaunchTimer t_q(h, 5, st);
            launch_k(quant_hidden_kernel, dim3(std::min(rows, h->sms * 8)), dim3(kQuantThreads), 0, st,
                     (const __nv_bfloat16*)hr, (const __nv_bfloat16*)hs, Tr, T, F, Fs, hq_r,
                     hq_r + (size_t)Tv * F, hsc_r, hsc_r + Tv);
            t_q.stop();
            L4MOE_CHECK_LAUNCH("hidden quantisation launch");
        }
    }

    LaunchTimer t_dn(h, 4, st);
    if (!fused) launch_gemm<MODE_DOWN, ET, WQ>(grid_for(dn_units), bm_dn, dn, st, small_tiles);
    {
        const long long n = (long long)T * d;
        // the routed planes then the shared ones; without experts only the shared
        launch_k(down_finish_kernel<ET>, dim3((int)std::min<long long>((n / 4 + 255) / 256, 8LL * h->sms)),
                 dim3(256), 0, st, (const float*)part, dn.part_stride_routed, E > 0 ? s_dn : 0,
                 (const float*)dn.part_shared, dn.part_stride_shared, s_dn, k, d, n, static_cast<ET*>(out),
                 done);
        ++h->launches;
    }
    t_dn.stop();
    L4MOE_CHECK_LAUNCH("down launch");
#undef L4MOE_CHECK_LAUNCH
    h->last_T = T;
    return L4MOE_OK;
}

// The column-scale pointers of 8-bit weights in the kernels' order: gate/up of
// experts 0..E-1, the shared gate/up, then the same for down.  Rewritten in
// place (the table never moves).
void fill_scale_table(l4moe_handle* h) {
    const int E = h->p.num_experts;
    for (int e = 0; e < E; ++e) {
        h->scale_tab[e] = h->s_gu[e];
        h->scale_tab[E + 1 + e] = h->s_dn[e];
    }
    h->scale_tab[E] = h->ss_gu;
    h->scale_tab[2 * E + 1] = h->ss_dn;
}

l4moe_status ensure_scales(l4moe_handle* h, cudaStream_t st) {
    const int E = h->p.num_experts;
    if (!h->d_scales) {
        cudaError_t e = cudaMalloc(&h->d_scales, sizeof(float*) * 2 * (E + 1));
        if (e != cudaSuccess) return cuda_fail(h, e, "scale table cudaMalloc");
        h->scales_dirty = true;
    }
    if (!h->scales_dirty) return L4MOE_OK;
    cudaError_t e = cudaMemcpyAsync(h->d_scales, h->scale_tab.data(), sizeof(float*) * h->scale_tab.size(),
                                    cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "scale table upload");
    h->scales_dirty = false;
    return L4MOE_OK;
}

l4moe_status check_forward_args(l4moe_handle* h, int T, const void* x, const void* Wr,
                                const void* const* Wgu, const void* const* Wdn, const void* Wsgu,
                                const void* Wsdn, const void* out) {
    if (!h) return L4MOE_ERR_ARG;
    if (T < 0) return fail(h, L4MOE_ERR_ARG, "T must be >= 0");
    int cur = -1;  // the workspace and descriptors live on the handle's device
    if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device)
        return fail(h, L4MOE_ERR_ARG, "the current CUDA device is not the handle's (the one current at l4moe_create)");
    const bool experts = h->p.num_experts > 0;  // without experts W_router, W_gate_up, W_down are unused
    if (!x || !Wsgu || !Wsdn || !out || (experts && (!Wr || !Wgu || !Wdn)))
        return fail(h, L4MOE_ERR_ARG, "null tensor pointer");
    const void* ptrs[] = {x, experts ? Wr : x, Wsgu, Wsdn, out};
    for (const void* q : ptrs)
        if (!aligned16(q)) return fail(h, L4MOE_ERR_ALIGN, "tensor pointer not 16-byte aligned");
    for (int e = 0; e < h->p.num_experts; ++e) {
        if (!Wgu[e] || !Wdn[e]) return fail(h, L4MOE_ERR_ARG, "null expert weight pointer");
        if (!aligned16(Wgu[e]) || !aligned16(Wdn[e]))
            return fail(h, L4MOE_ERR_ALIGN, "expert weight pointer not 16-byte aligned");
    }
    if (coded8(h->p.dtype) && !h->ss_gu)
        return fail(h, L4MOE_ERR_DTYPE, "8-bit weights need l4moe_set_weight_scales first");
    return L4MOE_OK;
}

l4moe_status forward_impl(l4moe_handle* h, int T, const void* x, const void* Wr,
                          const void* const* Wgu, const void* const* Wdn, const void* Wsgu,
                          const void* Wsdn, void* out, cudaStream_t st) {
    l4moe_status s;
    if ((s = ensure_workspace(h, T)) != L4MOE_OK) return s;
    if ((s = ensure_weight_maps(h, Wgu, Wdn, Wsgu, Wsdn, st)) != L4MOE_OK) return s;
    if (coded8(h->p.dtype) && (s = ensure_scales(h, st)) != L4MOE_OK) return s;
    switch (h->p.dtype) {
    case L4MOE_F32:
        return run_layer<float>(h, T, x, Wr, Wsgu, Wsdn, out, st, h->ws, h->ws_tokens, h->d_maps);
    case L4MOE_BF16:
        return run_layer<__nv_bfloat16>(h, T, x, Wr, Wsgu, Wsdn, out, st, h->ws, h->ws_tokens,
                                        h->d_maps);
    case L4MOE_FP8_E4M3:
        if (h->act8)
            return run_layer<__nv_bfloat16, kWqAct8>(h, T, x, Wr, Wsgu, Wsdn, out, st, h->ws, h->ws_tokens,
                                                     h->d_maps, h->d_scales);
        return run_layer<__nv_bfloat16, kWqE4M3>(h, T, x, Wr, Wsgu, Wsdn, out, st, h->ws, h->ws_tokens,
                                                 h->d_maps, h->d_scales);
    case L4MOE_INT8:
        return run_layer<__nv_bfloat16, kWqInt8>(h, T, x, Wr, Wsgu, Wsdn, out, st, h->ws, h->ws_tokens,
                                                 h->d_maps, h->d_scales);
    case L4MOE_INT4:
        return run_layer<__nv_bfloat16, kWqInt4>(h, T, x, Wr, Wsgu, Wsdn, out, st, h->ws, h->ws_tokens,
                                                 h->d_maps, h->d_scales);
    }
    return fail(h, L4MOE_ERR_DTYPE, "unknown dtype");
}

// ------------------------------------------------------------------------
// Allocation-free forward: workspace and weight descriptors in a fixed
// device array of this file, never in cudaMalloc'd memory.
static __device__ __align__(256) uint8_t g_static_ws[L4MOE_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
uint8_t* g_static_addr[kMaxDevices] = {};

// Device address of g_static_ws on the current device, resolved once per
// device (the host-side symbol is only a stand-in, not a device address).
l4moe_status static_workspace(l4moe_handle* h, uint8_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(h, L4MOE_ERR_UNSUPPORTED, "device index out of range");
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_addr[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_static_ws);
        if (e != cudaSuccess || !ptr) return cuda_fail(h, e, "cudaGetSymbolAddress(static workspace)");
        g_static_addr[dev] = static_cast<uint8_t*>(ptr);
    }
    *out = g_static_addr[dev];
    return L4MOE_OK;
}

}  // namespace

extern "C" {

l4moe_status l4moe_forward_static(l4moe_handle* h, int T, const void* x, const void* W_router,
                                  const void* const* W_gate_up, const void* const* W_down,
                                  const void* Ws_gate_up, const void* Ws_down, void* out,
                                  void* stream) {
    l4moe_status s = check_forward_args(h, T, x, W_router, W_gate_up, W_down, Ws_gate_up, Ws_down, out);
    if (s != L4MOE_OK || T == 0) return s;
    const int E = h->p.num_experts;
    const bool fp8 = coded8(h->p.dtype);
    const size_t ws_bytes = (ws_layout(h->p, T, h->sms, h->top_k, h->act8).device_total + 255) & ~size_t(255);
    const size_t maps_bytes = sizeof(CUtensorMap) * 2 * (E + 1);
    const size_t scales_bytes = fp8 ? sizeof(float*) * 2 * (E + 1) : 0;
    if (ws_bytes + maps_bytes + scales_bytes > L4MOE_STATIC_WORKSPACE_BYTES) {
        char msg[200];
        snprintf(msg, sizeof msg,
                 "T = %d needs %zu bytes of static workspace; the library's static array holds %u",
                 T, ws_bytes + maps_bytes + scales_bytes, (unsigned)L4MOE_STATIC_WORKSPACE_BYTES);
        return fail(h, L4MOE_ERR_WORKSPACE, msg);
    }
    uint8_t* base = nullptr;
    if ((s = static_workspace(h, &base)) != L4MOE_OK) return s;
    if ((s = encode_weight_maps(h, W_gate_up, W_down, Ws_gate_up, Ws_down)) != L4MOE_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    CUtensorMap* maps = reinterpret_cast<CUtensorMap*>(base + ws_bytes);
    // every call shares the array: upload this call's descriptors and clear
    // the state a forward expects to start at zero
    cudaError_t e = cudaMemcpyAsync(maps, h->h_maps.data(), maps_bytes, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "static descriptor upload");
    // the error word, the routing kernels' ticket and the fused GEMM's two
    // tile counters that follow it
    e = cudaMemsetAsync(base + ws_layout(h->p, T, h->sms, h->top_k, h->act8).err, 0, 4 * sizeof(unsigned), st);
    if (e != cudaSuccess) return cuda_fail(h, e, "static error word clear");
    const float* const* scales = nullptr;
    if (fp8) {  // the scale-pointer table of 8-bit weights follows the descriptors
        scales = reinterpret_cast<const float* const*>(base + ws_bytes + maps_bytes);
        e = cudaMemcpyAsync(const_cast<const float**>(scales), h->scale_tab.data(), scales_bytes,
                            cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) return cuda_fail(h, e, "static scale table upload");
    }
    const unsigned timing = h->timing;  // event timing would create events: off here
    h->timing = 0;
    if (h->p.dtype == L4MOE_F32)
        s = run_layer<float>(h, T, x, W_router, Ws_gate_up, Ws_down, out, st, base, T, maps);
    else if (h->p.dtype == L4MOE_FP8_E4M3 && h->act8)
        s = run_layer<__nv_bfloat16, kWqAct8>(h, T, x, W_router, Ws_gate_up, Ws_down, out, st, base, T, maps,
                                              scales);
    else if (h->p.dtype == L4MOE_FP8_E4M3)
        s = run_layer<__nv_bfloat16, kWqE4M3>(h, T, x, W_router, Ws_gate_up, Ws_down, out, st, base, T, maps,
                                              scales);
    else if (h->p.dtype == L4MOE_INT8)
        s = run_layer<__nv_bfloat16, kWqInt8>(h, T, x, W_router, Ws_gate_up, Ws_down, out, st, base, T, maps,
                                              scales);
    else if (h->p.dtype == L4MOE_INT4)
        s = run_layer<__nv_bfloat16, kWqInt4>(h, T, x, W_router, Ws_gate_up, Ws_down, out, st, base, T, maps,
                                              scales);
    else
        s = run_layer<__nv_bfloat16>(h, T, x, W_router, Ws_gate_up, Ws_down, out, st, base, T, maps);
    h->timing = timing;
    return s;
}

int l4moe_version(void) { return 100; }

const char* l4moe_status_string(l4moe_status s) {
    switch (s) {
    case L4MOE_OK: return "L4MOE_OK";
    case L4MOE_ERR_ARG: return "L4MOE_ERR_ARG";
    case L4MOE_ERR_DTYPE: return "L4MOE_ERR_DTYPE";
    case L4MOE_ERR_ALIGN: return "L4MOE_ERR_ALIGN";
    case L4MOE_ERR_CUDA: return "L4MOE_ERR_CUDA";
    case L4MOE_ERR_WORKSPACE: return "L4MOE_ERR_WORKSPACE";
    case L4MOE_ERR_TIMEOUT: return "L4MOE_ERR_TIMEOUT";
    case L4MOE_ERR_UNSUPPORTED: return "L4MOE_ERR_UNSUPPORTED";
    case L4MOE_ERR_RANGE: return "L4MOE_ERR_RANGE";
    }
    return "L4MOE_ERR_UNKNOWN";
}

l4moe_status l4moe_create(const l4moe_params* params, l4moe_handle** out) {
    if (!params || !out) return fail(nullptr, L4MOE_ERR_ARG, "null params or out");
    *out = nullptr;
    const l4moe_params& p = *params;
    if (p.dtype != L4MOE_F32 && p.dtype != L4MOE_BF16 && p.dtype != L4MOE_FP8_E4M3 && p.dtype != L4MOE_INT8 &&
        p.dtype != L4MOE_INT4)
        return fail(nullptr, L4MOE_ERR_DTYPE, "unknown dtype");
    if (p.d_model <= 0 || p.shared_ffn <= 0 || p.num_experts < 0 || p.num_experts > 256 ||
        p.expert_ffn < 0 || (p.num_experts > 0 && p.expert_ffn == 0))
        return fail(nullptr, L4MOE_ERR_ARG,
                    "shape out of range (need d, Fs > 0, 0 <= E <= 256, F > 0 when E > 0)");
    if (p.d_model % 64 || p.expert_ffn % 64 || p.shared_ffn % 64)
        return fail(nullptr, L4MOE_ERR_ALIGN, "d_model, expert_ffn and shared_ffn must be multiples of 64");
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(nullptr, L4MOE_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (major != 10 || minor != 0)
        return fail(nullptr, L4MOE_ERR_UNSUPPORTED, "this library is built for sm_100a (B200) only");
    if (!encode_fn()) return fail(nullptr, L4MOE_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled unavailable");
    l4moe_handle* h = new l4moe_handle();
    h->p = p;
    h->device = dev;
    h->sms = sms;
    h->h_maps.reserve(2 * (size_t)(p.num_experts + 1));
    h->scale_tab.assign(2 * (size_t)(p.num_experts + 1), nullptr);
    *out = h;
    return L4MOE_OK;
}

void l4moe_destroy(l4moe_handle* h) {
    if (!h) return;
    for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
    for (int b = 0; b < 2; ++b) {
        if (h->ev_h2d[b]) cudaEventDestroy(h->ev_h2d[b]);
        if (h->ev_comp[b]) cudaEventDestroy(h->ev_comp[b]);
        if (h->ev_d2h[b]) cudaEventDestroy(h->ev_d2h[b]);
    }
    if (h->s_in) cudaStreamDestroy(h->s_in);
    if (h->s_out) cudaStreamDestroy(h->s_out);
    for (auto& p : h->ev_pending) {
        cudaEventDestroy(p.second.first);
        cudaEventDestroy(p.second.second);
    }
    if (h->ws_owned && h->ws) cudaFree(h->ws);
    if (h->d_maps) cudaFree(h->d_maps);
    if (h->d_scales) cudaFree(h->d_scales);
    delete h;
}

size_t l4moe_workspace_size(const l4moe_handle* h, int max_tokens) {
    if (!h || max_tokens < 0) return 0;
    return ws_layout(h->p, max_tokens, h->sms, h->top_k, h->act8).total;
}

l4moe_status l4moe_set_top_k(l4moe_handle* h, int k) {
    if (!h) return L4MOE_ERR_ARG;
    const int E = h->p.num_experts;
    if (k < 1 || k > kMaxTopK || (E > 0 && k > E) || (E == 0 && k != 1))
        return fail(h, L4MOE_ERR_ARG, "top_k must be in [1, min(4, E)]");
    if (k == h->top_k) return L4MOE_OK;
    if (h->ws && !h->ws_owned && h->ws_bytes < ws_layout(h->p, h->ws_tokens, h->sms, k, h->act8).total)
        return fail(h, L4MOE_ERR_WORKSPACE, "the caller's workspace is too small for this top_k");
    if (h->ws && h->ws_owned) {  // re-laid out (and re-sized) by the next forward
        cudaError_t e = cudaFree(h->ws);  // synchronises: work in flight is done
        h->ws = nullptr;
        h->ws_tokens = 0;
        if (e != cudaSuccess) return cuda_fail(h, e, "workspace cudaFree");
    }
    h->top_k = k;
    return L4MOE_OK;
}

l4moe_status l4moe_set_act_fp8(l4moe_handle* h, int on) {
    if (!h) return L4MOE_ERR_ARG;
    if (on != 0 && on != 1) return fail(h, L4MOE_ERR_ARG, "act_fp8 must be 0 or 1");
    if (on && h->p.dtype != L4MOE_FP8_E4M3)
        return fail(h, L4MOE_ERR_DTYPE, "the FP8 activation mode needs E4M3 weights");
    const bool a = on != 0;
    if (a == h->act8) return L4MOE_OK;
    if (h->ws && !h->ws_owned && h->ws_bytes < ws_layout(h->p, h->ws_tokens, h->sms, h->top_k, a).total)
        return fail(h, L4MOE_ERR_WORKSPACE, "the caller's workspace is too small for the FP8 activation mode");
    if (h->ws && h->ws_owned) {  // re-laid out (and re-sized) by the next forward
        cudaError_t e = cudaFree(h->ws);  // synchronises: work in flight is done
        h->ws = nullptr;
        h->ws_tokens = 0;
        if (e != cudaSuccess) return cuda_fail(h, e, "workspace cudaFree");
    }
    // the weight descriptors' boxes differ: encode them again at the next forward
    h->h_maps.clear();
    h->hkey_sgu = h->hkey_sdn = nullptr;
    h->key_sgu = h->key_sdn = nullptr;
    h->act8 = a;
    return L4MOE_OK;
}

l4moe_status l4moe_set_workspace(l4moe_handle* h, void* dev_ptr, size_t bytes, int max_tokens) {
    if (!h) return L4MOE_ERR_ARG;
    if (!dev_ptr || max_tokens < 1) return fail(h, L4MOE_ERR_ARG, "null workspace or max_tokens < 1");
    if (reinterpret_cast<uintptr_t>(dev_ptr) & 255u)
        return fail(h, L4MOE_ERR_ALIGN, "workspace must be 256-byte aligned");
    if (bytes < ws_layout(h->p, max_tokens, h->sms, h->top_k, h->act8).total)
        return fail(h, L4MOE_ERR_WORKSPACE, "workspace smaller than l4moe_workspace_size");
    if (h->ws_owned && h->ws) cudaFree(h->ws);
    h->ws = static_cast<uint8_t*>(dev_ptr);
    h->ws_bytes = bytes;
    h->ws_tokens = max_tokens;
    h->ws_owned = false;
    cudaError_t e = cudaMemset(h->ws, 0, 256);
    if (e != cudaSuccess) return cuda_fail(h, e, "workspace cudaMemset");
    return L4MOE_OK;
}

l4moe_status l4moe_set_router_bias(l4moe_handle* h, const float* bias_dev) {
    if (!h) return L4MOE_ERR_ARG;
    if (bias_dev && (reinterpret_cast<uintptr_t>(bias_dev) & 3u))
        return fail(h, L4MOE_ERR_ALIGN, "bias must be 4-byte aligned");
    h->bias = bias_dev;
    return L4MOE_OK;
}

l4moe_status l4moe_set_weight_scales(l4moe_handle* h, const float* const* s_gate_up,
                                     const float* const* s_down, const float* ss_gate_up,
                                     const float* ss_down) {
    if (!h) return L4MOE_ERR_ARG;
    if (!coded8(h->p.dtype)) return fail(h, L4MOE_ERR_DTYPE, "scales apply to E4M3, int8 or int4 weights only");
    const int E = h->p.num_experts;
    if (!ss_gate_up || !ss_down || (E > 0 && (!s_gate_up || !s_down)))
        return fail(h, L4MOE_ERR_ARG, "null scale pointer");
    for (int e = 0; e < E; ++e)
        if (!s_gate_up[e] || !s_down[e]) return fail(h, L4MOE_ERR_ARG, "null expert scale pointer");
    h->s_gu.assign(s_gate_up, s_gate_up + (E > 0 ? E : 0));
    h->s_dn.assign(s_down, s_down + (E > 0 ? E : 0));
    h->ss_gu = ss_gate_up;
    h->ss_dn = ss_down;
    fill_scale_table(h);
    h->scales_dirty = true;
    return L4MOE_OK;
}

l4moe_status l4moe_set_fp8_scales(l4moe_handle* h, const float* const* s_gate_up,
                                  const float* const* s_down, const float* ss_gate_up,
                                  const float* ss_down) {
    return l4moe_set_weight_scales(h, s_gate_up, s_down, ss_gate_up, ss_down);
}

l4moe_status l4moe_forward(l4moe_handle* h, int T, const void* x, const void* W_router,
                           const void* const* W_gate_up, const void* const* W_down,
                           const void* Ws_gate_up, const void* Ws_down, void* out, void* stream) {
    l4moe_status s = check_forward_args(h, T, x, W_router, W_gate_up, W_down, Ws_gate_up, Ws_down, out);
    if (s != L4MOE_OK || T == 0) return s;
    return forward_impl(h, T, x, W_router, W_gate_up, W_down, Ws_gate_up, Ws_down, out,
                        static_cast<cudaStream_t>(stream));
}

l4moe_status l4moe_forward_host(l4moe_handle* h, int T, const void* x_host, const void* W_router,
                                const void* const* W_gate_up, const void* const* W_down,
                                const void* Ws_gate_up, const void* Ws_down, void* out_host,
                                void* stream) {
    l4moe_status s =
        check_forward_args(h, T, x_host, W_router, W_gate_up, W_down, Ws_gate_up, Ws_down, out_host);
    if (s != L4MOE_OK || T == 0) return s;
    if ((s = ensure_workspace(h, T)) != L4MOE_OK) return s;
    cudaError_t e;
    if (!h->s_in) {
        if ((e = cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(h, e, "copy stream creation");
        for (int b = 0; b < 2; ++b)
            if ((e = cudaEventCreateWithFlags(&h->ev_h2d[b], cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&h->ev_comp[b], cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&h->ev_d2h[b], cudaEventDisableTiming)) != cudaSuccess)
                return cuda_fail(h, e, "copy event creation");
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(h->p, h->ws_tokens, h->sms, h->top_k, h->act8);
    const size_t slab = (size_t)h->ws_tokens * h->p.d_model * act_bytes(h->p.dtype);
    const int b = h->host_slot;
    h->host_slot ^= 1;
    void* xin = h->ws + L.xin + b * slab;
    void* xout = h->ws + L.xout + b * slab;
    const size_t bytes = (size_t)T * h->p.d_model * act_bytes(h->p.dtype);
    // input copy on the copy-in stream, once the compute that last read this slot is done
    if (h->slot_used[b] && (e = cudaStreamWaitEvent(h->s_in, h->ev_comp[b], 0)) != cudaSuccess)
        return cuda_fail(h, e, "copy-in wait");
    if ((e = cudaMemcpyAsync(xin, x_host, bytes, cudaMemcpyHostToDevice, h->s_in)) != cudaSuccess)
        return cuda_fail(h, e, "input host-to-device copy");
    if ((e = cudaEventRecord(h->ev_h2d[b], h->s_in)) != cudaSuccess) return cuda_fail(h, e, "event record");
    // the layer on the caller's stream: after this input, and after the
    // output copy that last read this slot's output buffer
    if ((e = cudaStreamWaitEvent(st, h->ev_h2d[b], 0)) != cudaSuccess) return cuda_fail(h, e, "compute wait");
    if (h->slot_used[b] && (e = cudaStreamWaitEvent(st, h->ev_d2h[b], 0)) != cudaSuccess)
        return cuda_fail(h, e, "compute wait");
    if ((s = forward_impl(h, T, xin, W_router, W_gate_up, W_down, Ws_gate_up, Ws_down, xout, st)) != L4MOE_OK)
        return s;
    if ((e = cudaEventRecord(h->ev_comp[b], st)) != cudaSuccess) return cuda_fail(h, e, "event record");
    // output copy on the copy-out stream
    if ((e = cudaStreamWaitEvent(h->s_out, h->ev_comp[b], 0)) != cudaSuccess)
        return cuda_fail(h, e, "copy-out wait");
    if ((e = cudaMemcpyAsync(out_host, xout, bytes, cudaMemcpyDeviceToHost, h->s_out)) != cudaSuccess)
        return cuda_fail(h, e, "output device-to-host copy");
    if ((e = cudaEventRecord(h->ev_d2h[b], h->s_out)) != cudaSuccess) return cuda_fail(h, e, "event record");
    h->slot_used[b] = true;
    return L4MOE_OK;
}

l4moe_status l4moe_join_host(l4moe_handle* h, void* stream) {
    if (!h) return L4MOE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int b = 0; b < 2; ++b)
        if (h->slot_used[b]) {
            cudaError_t e = cudaStreamWaitEvent(st, h->ev_d2h[b], 0);
            if (e != cudaSuccess) return cuda_fail(h, e, "join wait");
        }
    return L4MOE_OK;
}

l4moe_status l4moe_get_routing(const l4moe_handle* h, const int32_t** idx, const float** gate,
                               const float** lmax, const float** margin, const int32_t** counts,
                               const int32_t** offsets, const int32_t** perm) {
    if (!h || !h->ws) return L4MOE_ERR_ARG;
    const WsLayout L = ws_layout(h->p, h->ws_tokens, h->sms, h->top_k, h->act8);
    if (idx) *idx = reinterpret_cast<const int32_t*>(h->ws + L.idx);
    if (gate) *gate = reinterpret_cast<const float*>(h->ws + L.gate);
    if (lmax) *lmax = reinterpret_cast<const float*>(h->ws + L.lmax);
    if (margin) *margin = reinterpret_cast<const float*>(h->ws + L.margin);
    if (counts) *counts = reinterpret_cast<const int32_t*>(h->ws + L.counts);
    if (offsets) *offsets = reinterpret_cast<const int32_t*>(h->ws + L.offsets);
    if (perm) *perm = reinterpret_cast<const int32_t*>(h->ws + L.perm);
    return L4MOE_OK;
}

l4moe_status l4moe_check_device_status(l4moe_handle* h, void* stream) {
    if (!h) return L4MOE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && h->s_out) e = cudaStreamSynchronize(h->s_out);
    if (e != cudaSuccess) return cuda_fail(h, e, "stream synchronize");
    if (!h->ws) return L4MOE_OK;
    unsigned word = 0;
    e = cudaMemcpy(&word, h->ws + ws_layout(h->p, h->ws_tokens, h->sms, h->top_k, h->act8).err, sizeof(word), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(h, e, "error word read");
    if (word == 0) return L4MOE_OK;
    cudaMemset(h->ws + ws_layout(h->p, h->ws_tokens, h->sms, h->top_k, h->act8).err, 0, sizeof(word));
    char msg[160];
    snprintf(msg, sizeof msg,
             "device error word 0x%x (1: producer wait, 2: MMA wait, 4: epilogue wait, 8: bad expert index, "
             "16: hidden value beyond f16)", word);
    return fail(h, (word & 7u) ? L4MOE_ERR_TIMEOUT : (word & 16u) ? L4MOE_ERR_RANGE : L4MOE_ERR_ARG, msg);
}

l4moe_status l4moe_selftest_wait(l4moe_handle* h, double limit_ms, void* stream) {
    if (!h) return L4MOE_ERR_ARG;
    if (!(limit_ms > 0.0 && limit_ms <= 1000.0)) return fail(h, L4MOE_ERR_ARG, "limit_ms must be in (0, 1000]");
    l4moe_status s;
    if ((s = ensure_workspace(h, 1)) != L4MOE_OK) return s;
    const WsLayout L = ws_layout(h->p, h->ws_tokens, h->sms, h->top_k, h->act8);
    unsigned* err = reinterpret_cast<unsigned*>(h->ws + L.err);
    wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, (uint64_t)(limit_ms * 1e6));
    ++h->launches;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(h, e, "self-test launch");
    return L4MOE_OK;
}

l4moe_status l4moe_set_timing(l4moe_handle* h, int mask) {
    if (!h || mask < 0 || mask >= (1 << L4MOE_NUM_KERNELS)) return L4MOE_ERR_ARG;
    h->timing = (unsigned)mask;
    return L4MOE_OK;
}

l4moe_status l4moe_read_timing(l4moe_handle* h, double* ms, uint64_t* launches) {
    if (!h || !ms || !launches) return L4MOE_ERR_ARG;
    if (h->ev_pending.empty()) return L4MOE_OK;
    cudaError_t e = cudaEventSynchronize(h->ev_pending.back().second.second);
    if (e != cudaSuccess) return cuda_fail(h, e, "timing event synchronize");
    for (auto& p : h->ev_pending) {
        float t = 0.f;
        e = cudaEventElapsedTime(&t, p.second.first, p.second.second);
        if (e != cudaSuccess) return cuda_fail(h, e, "timing elapsed time");
        ms[p.first] += t;
        launches[p.first] += 1;
        h->ev_pool.push_back(p.second.first);
        h->ev_pool.push_back(p.second.second);
    }
    h->ev_pending.clear();
    return L4MOE_OK;
}

const char* l4moe_kernel_name(int slot) {
    static const char* names[L4MOE_NUM_KERNELS] = {"router", "permute", "row_copy", "gemm_gate_up",
                                                   "gemm_down", "quant_hidden"};
    return (slot >= 0 && slot < L4MOE_NUM_KERNELS) ? names[slot] : "";
}

uint64_t l4moe_launch_count(const l4moe_handle* h) { return h ? h->launches : 0; }

l4moe_status l4moe_get_plan(const l4moe_handle* h, l4moe_plan* plan) {
    if (!h || !plan) return L4MOE_ERR_ARG;
    *plan = h->last_plan;
    return L4MOE_OK;
}

const char* l4moe_last_error(const l4moe_handle* h) {
    return h ? h->err.c_str() : g_create_error.c_str();
}

}  // extern "C"
