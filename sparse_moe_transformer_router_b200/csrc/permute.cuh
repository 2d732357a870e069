// permute.cuh -- token dispatch: per-expert histogram, exclusive scan,
// stable slot assignment, and the copy of the input rows into expert order.
//
// superteams.ai "Llama 4" glossary, routing sketch: each token is handed to
// the one expert its router picked.  On the GPU the tokens of each expert are
// gathered into a contiguous block of rows (expert-ordered "slots") so the
// experts run as a grouped GEMM.  The order inside an expert is by token
// index (stable), so slot = offsets[e] + #{t' < t : idx[t'] == e}.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "quant.cuh"
#include "schedule.cuh"
#include "topk.cuh"

namespace l4moe {

__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    return v;
}

// CTA-wide inclusive scan of N ints per thread, in thread order, and the
// CTA's totals.  Every thread of the CTA calls it (it synchronises).
template <int N>
__device__ void cta_incl_scan(int (&v)[N], int (&total)[N]) {
    __shared__ int sc[33 * N];  // warps' totals, their exclusive prefix, the CTA total
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int j = 0; j < N; ++j) v[j] = warp_incl_scan(v[j]);
    if (lane == 31)
#pragma unroll
        for (int j = 0; j < N; ++j) sc[warp * N + j] = v[j];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int j = 0; j < N; ++j) {
            const int t = lane < nw ? sc[lane * N + j] : 0;
            const int it = warp_incl_scan(t);
            if (lane < nw) sc[lane * N + j] = it - t;
            if (lane == 31) sc[32 * N + j] = it;
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < N; ++j) {
        v[j] += sc[warp * N + j];
        total[j] = sc[32 * N + j];
    }
    __syncthreads();  // sc free for the next call
}

// Both work lists (gate/up and down) from candidate groups [0, G), by every
// thread of the CTA: candidate g has rows(g), row0(g), expert(g), and
// ceil(rows / kTokTile) * fb_gu(g) gate/up tiles, ceil(rows / kTokTile) *
// fb_down down tiles (every fb >= 1).  Empty groups are left out; heavy
// groups (rows >= kHeavyRows) come first, each run in candidate order, so
// both lists hold the same groups at the same positions.  A pass of
// CTA-wide scans counts the heavy run; a second places every group.
template <typename RowsF, typename Row0F, typename ExpF, typename FbF>
__device__ void build_tables(GroupTable* tab_gu, GroupTable* tab_dn, int G, RowsF rows_of, Row0F row0_of,
                             ExpF exp_of, FbF fb_gu_of, int fb_down) {
    const int nt = blockDim.x;
    int heavy[3] = {0, 0, 0};  // the heavy run's groups, gate/up tiles, down tiles
    for (int base = 0; base < G; base += nt) {
        const int g = base + threadIdx.x;
        int v[3] = {0, 0, 0}, t[3];
        if (g < G) {
            const int rows = rows_of(g);
            if (rows >= kHeavyRows) {
                const int ntb = (rows + kTokTile - 1) / kTokTile;
                v[0] = 1;
                v[1] = ntb * fb_gu_of(g);
                v[2] = ntb * fb_down;
            }
        }
        cta_incl_scan<3>(v, t);
#pragma unroll
        for (int j = 0; j < 3; ++j) heavy[j] += t[j];
    }
    int carry[6] = {0, 0, 0, 0, 0, 0};  // groups, gate/up tiles, down tiles: heavy run, then light run
    for (int base = 0; base < G; base += nt) {
        const int g = base + threadIdx.x;
        int rows = 0, tg = 0, td = 0;
        bool hv = false;
        if (g < G) {
            rows = rows_of(g);
            if (rows > 0) {
                const int ntb = (rows + kTokTile - 1) / kTokTile;
                tg = ntb * fb_gu_of(g);
                td = ntb * fb_down;
                hv = rows >= kHeavyRows;
            }
        }
        const bool in = rows > 0;
        int v[6] = {in && hv ? 1 : 0, in && hv ? tg : 0, in && hv ? td : 0,
                    in && !hv ? 1 : 0, in && !hv ? tg : 0, in && !hv ? td : 0};
        int t[6];
        cta_incl_scan<6>(v, t);
        if (in) {  // this group's run: selects, not an index (keeps the arrays in registers)
            const int pos = (hv ? carry[0] + v[0] : heavy[0] + carry[3] + v[3]) - 1;
            const int sg = (hv ? carry[1] + v[1] : heavy[1] + carry[4] + v[4]) - tg;
            const int sd = (hv ? carry[2] + v[2] : heavy[2] + carry[5] + v[5]) - td;
            const int r0 = row0_of(g), ex = exp_of(g);
            tab_gu->rows[pos] = rows;
            tab_gu->row0[pos] = r0;
            tab_gu->expert[pos] = ex;
            tab_gu->tile_start[pos] = sg;
            tab_dn->rows[pos] = rows;
            tab_dn->row0[pos] = r0;
            tab_dn->expert[pos] = ex;
            tab_dn->tile_start[pos] = sd;
        }
#pragma unroll
        for (int j = 0; j < 6; ++j) carry[j] += t[j];
    }
    if (threadIdx.x == 0) {
        const int n = carry[0] + carry[3];
        tab_gu->num_groups = n;
        tab_gu->heavy_tiles = carry[1];
        tab_gu->total_tiles = carry[1] + carry[4];
        tab_gu->tile_start[n] = carry[1] + carry[4];
        tab_dn->num_groups = n;
        tab_dn->heavy_tiles = carry[2];
        tab_dn->total_tiles = carry[2] + carry[5];
        tab_dn->tile_start[n] = carry[2] + carry[5];
    }
}

// Stable ranks inside one chunk of entries, thread i of the CTA holding the
// chunk's entry i with expert e (-1: none).  Returns the entry's rank among
// the chunk's entries of its expert held by lower threads (-1 for none) and
// writes the chunk's per-expert counts to chunk_row[E].  A warp's
// __match_any_sync groups its entries by expert; a prefix over the warps,
// per expert, orders the groups.  smem: wcnt[warps][E] ints.
__device__ int chunk_rank(int e, int E, int* wcnt, int32_t* __restrict__ chunk_row) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    for (int i = tid; i < nwarps * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int lane_rank = __popc(same & ((1u << lane) - 1u));
    if (e >= 0 && lane_rank == 0) wcnt[warp * E + e] = __popc(same);
    __syncthreads();
    for (int x = tid; x < E; x += blockDim.x) {  // prefix over warps, per expert
        int acc = 0;
        for (int w = 0; w < nwarps; ++w) {
            const int v = wcnt[w * E + x];
            wcnt[w * E + x] = acc;
            acc += v;
        }
        chunk_row[x] = acc;
    }
    __syncthreads();
    return e >= 0 ? wcnt[warp * E + e] + lane_rank : -1;
}

// The final step of a chunked dispatch, run by one CTA once every chunk's
// per-expert counts are in chunk_base[chunks][E] and visible to it: each
// count becomes its chunk's first slot for the expert (offsets[e] plus the
// expert's entries in earlier chunks), and counts[E], offsets[E + 1] and the
// two work lists are written.  Any CTA size that is a multiple of 32.
// The counts are staged in shared memory a block of experts at a time, each
// thread's loads of a pass issued before any is stored (one L2 round trip
// per pass, not per element); tpe consecutive threads scan one expert, each
// a run of consecutive chunks, joined by a segmented shuffle scan; warp 0
// then scans over the experts, and the whole CTA writes the lists
// (build_tables).
// smem: tot[E], soff[E + 1] and stage[cap] ints, cap >= chunks, stage and
// chunk_base 16-byte aligned.  U: 4-byte loads in flight per thread (2U
// 16-byte ones): more for a small CTA, fewer where registers are scarce.
template <int U>
__device__ void dispatch_finish(int32_t* chunk_base, int chunks, int T, int E, int fb_gu_routed,
                                int fb_gu_shared, int fb_down, int32_t* __restrict__ counts,
                                int32_t* __restrict__ offsets, GroupTable* tab_gu, GroupTable* tab_dn,
                                int* tot, int* soff, int* stage, int cap) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x;
    // threads per expert: a power of two, at most a warp
    int tpe = 1;
    while (tpe < 32 && 2 * tpe * E <= nt) tpe *= 2;
    const int xblk = max(1, min(E, cap / chunks));  // experts per staged block
    const int per = (chunks + tpe - 1) / tpe;        // chunks per thread
    const int seg = lane & ~(tpe - 1);               // first lane of this thread's segment
    const bool whole = xblk >= E;                    // every expert staged at once: no write-back pass
    for (int x0 = 0; x0 < E; x0 += xblk) {
        const int xe = min(xblk, E - x0);
        const int n = chunks * xe;
        if (whole && (E & 3) == 0) {  // [chunks][E] as it lies in memory: 16-byte loads, 2U in flight
            const int n4 = n >> 2;
            const int4* src = reinterpret_cast<const int4*>(chunk_base);
            int4* dst = reinterpret_cast<int4*>(stage);
            for (int i0 = 0; i0 < n4; i0 += 2 * U * nt) {
                int4 v[2 * U];
#pragma unroll
                for (int j = 0; j < 2 * U; ++j) {
                    const int i = i0 + j * nt + tid;
                    if (i < n4) v[j] = __ldcg(src + i);
                }
#pragma unroll
                for (int j = 0; j < 2 * U; ++j) {
                    const int i = i0 + j * nt + tid;
                    if (i < n4) dst[i] = v[j];
                }
            }
        } else {
            for (int i0 = 0; i0 < n; i0 += U * nt) {
                int v[U];
#pragma unroll
                for (int j = 0; j < U; ++j) {
                    const int i = i0 + j * nt + tid;
                    const int c = i / xe;
                    v[j] = i < n ? __ldcg(chunk_base + (size_t)c * E + x0 + (i - c * xe)) : 0;
                }
#pragma unroll
                for (int j = 0; j < U; ++j) {
                    const int i = i0 + j * nt + tid;
                    if (i < n) stage[i] = v[j];
                }
            }
        }
        __syncthreads();
        for (int xx0 = 0; xx0 < xe; xx0 += nt / tpe) {
            const int xx = xx0 + tid / tpe;  // this thread's expert (block-relative)
            const int part = tid & (tpe - 1);
            const int c0 = min(chunks, part * per), c1 = min(chunks, c0 + per);
            int s = 0;
            if (xx < xe) {
#pragma unroll 8
                for (int c = c0; c < c1; ++c) s += stage[c * xe + xx];
            }
            int incl = s;  // inclusive scan over the expert's tpe threads
            for (int off = 1; off < tpe; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off, tpe);
                if ((lane - seg) >= off) incl += o;
            }
            int acc = incl - s;
            if (xx < xe) {
#pragma unroll 8
                for (int c = c0; c < c1; ++c) {
                    const int v = stage[c * xe + xx];
                    stage[c * xe + xx] = acc;
                    acc += v;
                }
                if (part == tpe - 1) tot[x0 + xx] = incl;
            }
        }
        __syncthreads();
        if (!whole) {  // the block's prefixes back to the chunk bases (the offsets follow)
            for (int i = tid; i < n; i += nt) {
                const int c = i / xe, x = i - c * xe;
                chunk_base[(size_t)c * E + x0 + x] = stage[i];
            }
            __syncthreads();
        }
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the counts (up to 8 experts per lane)
        int local[8];
        int sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int x = lane * 8 + j;
            local[j] = (x < E) ? tot[x] : 0;
            sum += local[j];
        }
        const int incl = warp_incl_scan(sum);
        int acc = incl - sum;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int x = lane * 8 + j;
            if (x < E) {
                soff[x] = acc;
                offsets[x] = acc;
                counts[x] = local[j];
            }
            acc += local[j];
        }
        if (lane == 31) {
            soff[E] = incl;
            offsets[E] = incl;
        }
    }
    __syncthreads();
    if (whole && (E & 3) == 0) {  // stage is [chunks][E]: 16-byte stores
        const int4* src = reinterpret_cast<const int4*>(stage);
        int4* dst = reinterpret_cast<int4*>(chunk_base);
        for (int i = tid; i < (chunks * E) >> 2; i += nt) {
            const int x = (4 * i) % E;
            const int4 v = src[i];
            dst[i] = make_int4(v.x + soff[x], v.y + soff[x + 1], v.z + soff[x + 2], v.w + soff[x + 3]);
        }
    } else if (whole) {
        for (int i = tid; i < chunks * E; i += nt) chunk_base[i] = stage[i] + soff[i % E];
    } else {
        for (int i0 = 0; i0 < chunks * E; i0 += U * nt) {
            int v[U];
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int i = i0 + j * nt + tid;
                v[j] = i < chunks * E ? chunk_base[i] : 0;
            }
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int i = i0 + j * nt + tid;
                if (i < chunks * E) chunk_base[i] = v[j] + soff[i % E];
            }
        }
    }
    // candidate 0 is the shared expert, 1..E the routed experts
    build_tables(
        tab_gu, tab_dn, E + 1, [&](int g) { return g == 0 ? T : tot[g - 1]; },
        [&](int g) { return g == 0 ? 0 : soff[g - 1]; }, [&](int g) { return g == 0 ? E : g - 1; },
        [&](int g) { return g == 0 ? fb_gu_shared : fb_gu_routed; }, fb_down);
}

// Work lists of a layer without experts: one group (the shared SwiGLU, as
// expert 0 == num_experts) over the T tokens in order.  One warp.
__global__ void dense_table_kernel(GroupTable* tab_gu, GroupTable* tab_dn, int T, int fb_gu, int fb_dn) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    if (threadIdx.x >= 32) return;
    const int tb = (T + kTokTile - 1) / kTokTile;
    for (int w = 0; w < 2; ++w) {
        GroupTable* tab = w == 0 ? tab_gu : tab_dn;
        const int tiles = tb * (w == 0 ? fb_gu : fb_dn);
        if (lane == 0) {
            tab->num_groups = T > 0 ? 1 : 0;
            tab->total_tiles = tiles;
            tab->heavy_tiles = T >= kHeavyRows ? tiles : 0;
            tab->rows[0] = T;
            tab->row0[0] = 0;
            tab->expert[0] = 0;
            tab->tile_start[0] = 0;
            tab->tile_start[1] = tiles;
        }
    }
}

// Single CTA of 1024 threads.  Writes counts[E], offsets[E+1], perm[T]
// (slot -> token), inv[T] (token -> slot) and two work lists:
//   tab_gu : shared expert (rows T) then the routed experts, gate/up GEMM
//   tab_dn : shared expert (rows T, token order) then the routed experts,
//            down GEMM (the two contractions meet in fp32 partials)
// smem: wcnt[32][E] + running[E] ints.
//
// Top-k (k >= 1): each token owns k entries n = t * k + j (its j-th
// selected expert), and the routed rows are these T * k entries: idx, gate,
// inv are [T * k], perm maps a slot to its entry, and the routed groups'
// rows add up to T * k while the shared expert keeps its T token rows.
//
// logits != null (expert-split router, logits [T][E] biased fp32): first
// finish the routing here -- per token, the k largest of the E logits
// (lower index first on ties, NaN never selected), the margin of the k-th
// to the next one and the sigmoid gates -- writing idx, gate, lmax, margin.
__global__ void __launch_bounds__(1024) permute_kernel(const float* __restrict__ logits,
                                                       float* __restrict__ gate,
                                                       float* __restrict__ lmax,
                                                       float* __restrict__ margin,
                                                       int32_t* __restrict__ idx, int T, int k,
                                                       int E, int fb_gu_routed, int fb_gu_shared,
                                                       int fb_down, int32_t* __restrict__ counts,
                                                       int32_t* __restrict__ offsets,
                                                       int32_t* __restrict__ perm,
                                                       int32_t* __restrict__ inv,
                                                       GroupTable* tab_gu, GroupTable* tab_dn,
                                                       unsigned* err) {
    pdl_enter();
    extern __shared__ int psm[];
    int* wcnt = psm;              // [32][E]
    int* running = psm + 32 * E;  // [E]
    int* soff = running + E;      // [E + 1]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (logits) {
        // one warp per token: lane owns experts lane, lane+32, ... (ascending
        // inside the lane, so each lane's list is in selection order); the
        // warp then takes k + 1 heads, each the first by (value, then index)
        for (int t = warp; t < T; t += 32) {
            TopK tk;
            tk.init();
            for (int e = lane; e < E; e += 32) tk.offer(logits[(size_t)t * E + e], e);
            TopK out;
            out.init();
            int pos = 0;  // entries of this lane's list already taken
#pragma unroll
            for (int j = 0; j <= kMaxTopK; ++j) {
                float hv = tk.value(pos);
                int hi = pos <= kMaxTopK ? tk.index(pos) : -1;
                int hl = lane;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, hv, off);
                    const int oi = __shfl_xor_sync(0xffffffffu, hi, off);
                    const int ol = __shfl_xor_sync(0xffffffffu, hl, off);
                    if (topk_before(ov, oi, hv, hi)) {
                        hv = ov;
                        hi = oi;
                        hl = ol;
                    }
                }
                out.set(j, hv, hi);
                if (hl == lane && hi >= 0) ++pos;
            }
            if (lane == 0) {
                out.fill_empty(k);
#pragma unroll
                for (int j = 0; j < kMaxTopK; ++j) {
                    if (j < k) {
                        const size_t n = (size_t)t * k + j;
                        idx[n] = out.index(j);
                        lmax[n] = out.value(j);
                        gate[n] = 1.0f / (1.0f + expf(-out.value(j)));
                    }
                }
                margin[t] = out.value(k - 1) - out.value(k);
            }
        }
        __syncthreads();
    }
    const int Tv = T * k;  // entries: token t's j-th expert is entry t * k + j
    for (int e = tid; e < E; e += 1024) running[e] = 0;
    __syncthreads();
    for (int c0 = 0; c0 < Tv; c0 += 1024) {
        for (int i = tid; i < 32 * E; i += 1024) wcnt[i] = 0;
        __syncthreads();
        const int t = c0 + tid;
        int e = -1;
        if (t < Tv) {
            e = idx[t];
            if (e < 0 || e >= E) {
                atomicOr(err, DEV_ERR_BAD_INDEX);
                e = -1;
            }
        }
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int lane_rank = __popc(same & ((1u << lane) - 1u));
        if (e >= 0 && lane_rank == 0) wcnt[warp * E + e] = __popc(same);
        __syncthreads();
        for (int x = tid; x < E; x += 1024) {  // prefix over warps, per expert
            int acc = running[x];
            for (int w = 0; w < 32; ++w) {
                const int v = wcnt[w * E + x];
                wcnt[w * E + x] = acc;
                acc += v;
            }
            running[x] = acc;
        }
        __syncthreads();
        if (t < Tv) inv[t] = e >= 0 ? wcnt[warp * E + e] + lane_rank : -1;  // rank inside expert
        __syncthreads();
    }
    // exclusive scan of the counts (warp 0, up to 8 experts per lane)
    if (warp == 0) {
        int local[8];
        int sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            local[j] = (e < E) ? running[e] : 0;
            sum += local[j];
        }
        const int incl = warp_incl_scan(sum);
        int acc = incl - sum;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            if (e < E) {
                soff[e] = acc;
                offsets[e] = acc;
                counts[e] = local[j];
            }
            acc += local[j];
        }
        if (lane == 31) {
            soff[E] = incl;
            offsets[E] = incl;
        }
    }
    __syncthreads();
    for (int t = tid; t < Tv; t += 1024) {
        const int e = idx[t];
        if (e >= 0 && e < E) {
            const int slot = soff[e] + inv[t];
            inv[t] = slot;
            perm[slot] = t;
        }
    }
    // candidate 0 is the shared expert, 1..E the routed experts
    build_tables(
        tab_gu, tab_dn, E + 1, [&](int g) { return g == 0 ? T : running[g - 1]; },
        [&](int g) { return g == 0 ? 0 : soff[g - 1]; }, [&](int g) { return g == 0 ? E : g - 1; },
        [&](int g) { return g == 0 ? fb_gu_shared : fb_gu_routed; }, fb_down);
}

// Multi-CTA dispatch of a batch whose routing is already in idx[T * k]: CTA
// c ranks the kDispatchChunk entries [c * kDispatchChunk, ...) -- a warp's
// __match_any_sync groups its entries by expert, a prefix over the 32 warps
// orders the groups -- and writes each entry's rank inside its expert and
// chunk to inv[n] and the chunk's per-expert counts to chunk_base[c][E].  The
// last CTA to finish (atomic ticket after a memory fence, no waiting) turns
// the counts into chunk bases (offsets[e] + entries of e in earlier chunks),
// writes counts[E], offsets[E + 1] and the two work lists, and resets the
// ticket.  A slot is then chunk_base[c][e] + inv[n] (permute_rows_kernel):
// the stable expert order, as the single-CTA permute_kernel gives it.
// smem: wcnt[max(32 * E, chunks)] + tot[E] + soff[E + 1] ints.
constexpr int kDispatchChunk = 1024;
// Chunks of either dispatch of n entries: dispatch_kernel's of kDispatchChunk
// entries, or a dispatching router's of 128 / S tokens (S <= 8 K slices,
// 128-token tiles, the last one ragged), whichever are more.
__host__ __device__ constexpr size_t router_max_chunks(size_t n) {
    return 8 * ((n + 127) / 128) > (n + kDispatchChunk - 1) / kDispatchChunk ? 8 * ((n + 127) / 128)
                                                                              : (n + kDispatchChunk - 1) / kDispatchChunk;
}

__global__ void __launch_bounds__(kDispatchChunk) dispatch_kernel(
    const int32_t* __restrict__ idx, int T, int k, int E, int fb_gu_routed, int fb_gu_shared, int fb_down,
    int32_t* __restrict__ chunk_base, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ inv, GroupTable* tab_gu, GroupTable* tab_dn, unsigned* ticket, unsigned* err) {
    pdl_enter();
    extern __shared__ __align__(16) int dsm[];
    const int stage_n = max(32 * E, (int)gridDim.x);  // wcnt, then the last CTA's staging (a row per chunk)
    int* wcnt = dsm;           // [32][E]
    int* tot = dsm + stage_n;  // [E]
    int* soff = tot + E;       // [E + 1]
    __shared__ unsigned s_last;
    const int tid = threadIdx.x;
    const int Tv = T * k;
    const int chunks = gridDim.x;
    const int n = blockIdx.x * kDispatchChunk + tid;
    int e = -1;
    if (n < Tv) {
        e = idx[n];
        if (e < 0 || e >= E) {
            atomicOr(err, DEV_ERR_BAD_INDEX);
            e = -1;
        }
    }
    const int r = chunk_rank(e, E, wcnt, chunk_base + (size_t)blockIdx.x * E);
    if (n < Tv) inv[n] = r;

    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(ticket, 1u) == (unsigned)chunks - 1u) ? 1u : 0u;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // last CTA: the chunk bases, counts, offsets and work lists (the warps'
    // count rows are free now and stage the chunks' counts)
    dispatch_finish<2>(chunk_base, chunks, T, E, fb_gu_routed, fb_gu_shared, fb_down, counts, offsets, tab_gu,
                       tab_dn, tot, soff, wcnt, stage_n);
    if (tid == 0) *ticket = 0u;
}

// Expert-ordered copy of the input rows, xp[inv[n]] = x[n / k] for each
// entry n, and the gate of each slot, gate_slot[inv[n]] = gate[n].  The sigmoid gate scales the
// routed expert's input, which is linear in the gate/up contraction, so it
// is applied to the fp32 accumulator in the GEMM epilogue instead of
// rounding g * x to the activation type here.  OT = IT copies exactly; for
// E4M3 layers IT = bf16, OT = f16 (the contractions' operand type) and
// x_tok (if not null) also receives the f16 rows in token order.  inv ==
// null keeps token order (and gate / gate_slot are then unused).
// One warp per token row, 16-byte vectors; d % 8 == 0.
// inv_s: the reciprocal of the row's power-of-two scale (f16_row_scale).
__device__ __forceinline__ uint4 cvt_row_vec(uint4 v, __nv_bfloat16, __half, float inv_s = 1.0f) {
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        const __half2 hv = __floats2half2_rn(f.x * inv_s, f.y * inv_s);
        w[i] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}
template <typename T>
__device__ __forceinline__ uint4 cvt_row_vec(uint4 v, T, T, float = 1.0f) { return v; }

// Layers with 8-bit weights hold x in f16 for their contractions.  A row
// whose largest |x| is beyond f16's largest finite value (65504) is divided
// by a power of two that brings it inside -- exact, only the exponents
// change -- and the row's fp32 accumulators are multiplied back by it in the
// gate/up epilogue (with the sigmoid gate for routed rows).  Rows in range,
// and rows holding inf or NaN, keep the scale 1.
__device__ __forceinline__ float f16_row_scale(float amax) {
    if (!(amax > 65504.0f) || !(amax < INFINITY)) return 1.0f;
    int e;
    frexpf(amax / 65504.0f, &e);  // amax / 65504 < 2^e
    return ldexpf(1.0f, e);
}

// The scale of a token row converted from IT to OT: the power-of-two f16
// range scale (8-bit weight layers), or the E4M3 row scale (FP8 activation
// mode, OT = uint8_t codes).
template <typename IT, typename OT>
__device__ __forceinline__ float row_scale_of(float amax) {
    if constexpr (std::is_same<OT, uint8_t>::value) return e4m3_row_scale(amax);
    else return f16_row_scale(amax);
}

// 16 bytes of an input row (vector c) -> the same elements of the output
// row: copied, divided by the power-of-two scale q.s into f16 (times its
// reciprocal, exact for a power of two), or quantised to E4M3 codes with the
// row scale q.s (8 bytes).
template <typename IT, typename OT>
__device__ __forceinline__ void put_row_vec(OT* orow, int c, uint4 v, const RowScale& q) {
    if constexpr (std::is_same<OT, uint8_t>::value)
        reinterpret_cast<uint2*>(orow)[c] = bf16x8_to_e4m3(v, q);
    else
        reinterpret_cast<uint4*>(orow)[c] = cvt_row_vec(v, IT{}, OT{}, q.r);
}

// chunk_base (not null, after dispatch_kernel or a dispatching router):
// inv[n] holds the entry's rank inside its expert and chunk (chunk entries
// per chunk); its slot is chunk_base[n / chunk][idx[n]] + inv[n], which this
// kernel writes back to inv[n] and records in perm.
// tokscale (8-bit weight layers; not null): each token's row scale (the
// power-of-two f16 range scale, or the E4M3 scale when OT is uint8_t codes),
// written once per token; gate_slot then carries gate * scale.
template <typename IT, typename OT>
__global__ void __launch_bounds__(256) permute_rows_kernel(const IT* __restrict__ x,
                                                           const float* __restrict__ gate,
                                                           int32_t* __restrict__ inv,
                                                           int T, int k, int d, OT* __restrict__ xp,
                                                           float* __restrict__ gate_slot,
                                                           OT* __restrict__ x_tok,
                                                           const int32_t* __restrict__ idx,
                                                           const int32_t* __restrict__ chunk_base, int chunk,
                                                           int E,
                                                           int32_t* __restrict__ perm,
                                                           float* __restrict__ tokscale) {
    pdl_enter();
    static_assert(sizeof(IT) == sizeof(OT) || std::is_same<OT, uint8_t>::value,
                  "row copy keeps the element size unless it quantises");
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    // one warp per entry n = t * k + j (token t's j-th expert)
    for (int n = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; n < T * k; n += warps) {
        const int t = n / k;
        int slot = inv ? inv[n] : n;
        if (chunk_base) {
            if (lane == 0) {
                const int e = idx[n];
                slot = (slot >= 0 && e >= 0 && e < E) ? chunk_base[(size_t)(n / chunk) * E + e] + slot : -1;
                if (slot >= 0 && slot < T * k) {
                    inv[n] = slot;
                    perm[slot] = n;
                }
            }
            slot = __shfl_sync(0xffffffffu, slot, 0);
        }
        if (slot < 0 || slot >= T * k) continue;  // an entry the permutation rejected (bad expert index)
        const uint4* s = reinterpret_cast<const uint4*>(x + (size_t)t * d);
        OT* o = xp + (size_t)slot * d;
        OT* ot = (x_tok && n % k == 0) ? x_tok + (size_t)t * d : nullptr;
        const int nv = d * (int)sizeof(IT) / 16;
        float sc = 1.0f;  // the row's scale (converted rows of 8-bit weight layers)
        if constexpr (!std::is_same<IT, OT>::value) {
            float m = 0.0f;
            for (int i = lane; i < nv; i += 32) m = absmax_vec(s[i], m);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            sc = row_scale_of<IT, OT>(m);
            if (lane == 0 && tokscale && n % k == 0) tokscale[t] = sc;
        }
        if (lane == 0 && gate_slot) gate_slot[slot] = gate[n] * sc;
        const RowScale q = row_scale(sc);
        // four 16-byte loads per lane in flight before any store
        for (int i0 = lane; i0 < nv; i0 += 4 * 32) {
            uint4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (i0 + 32 * j < nv) v[j] = s[i0 + 32 * j];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (i0 + 32 * j >= nv) continue;
                put_row_vec<IT, OT>(o, i0 + 32 * j, v[j], q);
                if (ot) put_row_vec<IT, OT>(ot, i0 + 32 * j, v[j], q);
            }
        }
    }
}

}  // namespace l4moe
