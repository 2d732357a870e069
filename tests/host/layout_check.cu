// Host-side check of the library's workspace layout and split-K plan
// (csrc/l4moe.cu, compiled into this program): for random layer shapes,
// dtypes (E4M3 with and without the FP8 activation mode), experts per
// token, SM counts and token budgets, every workspace
// segment is 256-byte aligned, in order and large enough for any batch of at
// most the budgeted tokens -- in particular the fp32 partial planes of the
// split-K plan a batch of T tokens gets -- and every k-range of a split keeps
// at least 8 k-blocks; the tensor-core router's stages, slice exchange and
// dispatch staging fit its shared memory.  Prints "OK <cases>" or the first
// violation.
#include <cstdio>
#include <random>

#include "l4moe.cu"

namespace {

bool g_act8 = false;  // the case being checked is in the FP8 activation mode

bool fail_case(const char* what, const l4moe_params& p, int T, int k, int sms) {
    printf("BAD %s: d %d F %d Fs %d E %d dtype %d act8 %d T %d k %d sms %d\n", what, p.d_model, p.expert_ffn,
           p.shared_ffn, p.num_experts, (int)p.dtype, (int)g_act8, T, k, sms);
    return false;
}

bool check(const l4moe_params& p, int Tmax, int k, int sms, bool act8 = false) {
    g_act8 = act8;
    const WsLayout L = ws_layout(p, Tmax, sms, k, act8);
    const size_t seg[] = {L.err, L.idx, L.gate, L.lmax, L.margin, L.inv, L.perm, L.gslot, L.counts, L.offsets,
                          L.chunk, L.tab_gu, L.tab_dn, L.xg, L.hr, L.hs, L.x16, L.xsc, L.hq, L.hsc, L.part,
                          L.logits, L.device_total,
                          L.xin, L.xout, L.total};
    const int nseg = sizeof(seg) / sizeof(seg[0]);
    for (int i = 0; i < nseg; ++i) {
        if (seg[i] % 256) return fail_case("segment not 256-aligned", p, Tmax, k, sms);
        if (i && seg[i] < seg[i - 1]) return fail_case("segments out of order", p, Tmax, k, sms);
    }
    auto size_of = [&](size_t off) {  // bytes up to the next segment
        for (int i = 0; i + 1 < nseg; ++i)
            if (seg[i] == off) {
                size_t j = i + 1;
                while ((int)j < nseg - 1 && seg[j] == off) ++j;
                return seg[j] - off;
            }
        return (size_t)0;
    };
    const size_t t = (size_t)Tmax, tv = t * k, E = p.num_experts, a = act_bytes(p.dtype);
    const size_t d = p.d_model, F = p.expert_ffn, Fs = p.shared_ffn;
    if (size_of(L.idx) < 4 * tv || size_of(L.gate) < 4 * tv || size_of(L.lmax) < 4 * tv ||
        size_of(L.inv) < 4 * tv || size_of(L.perm) < 4 * tv || size_of(L.gslot) < 4 * tv ||
        size_of(L.margin) < 4 * t)
        return fail_case("routing vectors too small", p, Tmax, k, sms);
    if ((E && size_of(L.counts) < 4 * E) || size_of(L.offsets) < 4 * (E + 1))
        return fail_case("counts / offsets too small", p, Tmax, k, sms);
    if (size_of(L.tab_gu) < sizeof(GroupTable) || size_of(L.tab_dn) < sizeof(GroupTable))
        return fail_case("work lists too small", p, Tmax, k, sms);
    if ((E && size_of(L.xg) < tv * d * a) || (E && size_of(L.hr) < tv * F * a) || size_of(L.hs) < t * Fs * a)
        return fail_case("activation rows too small", p, Tmax, k, sms);
    if (coded8(p.dtype) && size_of(L.x16) < t * d * 2) return fail_case("f16 x too small", p, Tmax, k, sms);
    if (coded8(p.dtype) && size_of(L.xsc) < 4 * t) return fail_case("row scales too small", p, Tmax, k, sms);
    // FP8 activation mode: hidden codes (routed [T k][F] then shared [T][Fs]) and row scales
    if (act8 && (size_of(L.hq) < tv * F + t * Fs || size_of(L.hsc) < 4 * (tv + t)))
        return fail_case("hidden codes / scales too small", p, Tmax, k, sms);
    if (E && size_of(L.logits) < 4 * std::min<size_t>(t, 128) * E)
        return fail_case("router logits too small", p, Tmax, k, sms);
    // the small-batch routing's partial logits [slices][T][E] for T <= kSmallMaxTokens
    const size_t slices = (d + kSmallSliceK - 1) / kSmallSliceK;
    if (E && size_of(L.logits) < 4 * slices * std::min<size_t>(t, kSmallMaxTokens) * E)
        return fail_case("small-batch partial logits too small", p, Tmax, k, sms);
    // the dispatch chunk bases [chunks][E]: up to 8 chunks per 128-token tile (the router's)
    if (E && size_of(L.chunk) < 4 * 8 * ((tv + 127) / 128) * E)
        return fail_case("dispatch chunk bases too small", p, Tmax, k, sms);
    if (L.xout + 2 * t * d * a > L.total || L.xin + 2 * t * d * a > L.xout)
        return fail_case("host staging too small", p, Tmax, k, sms);
    const int kblk = act8 ? 128 : (int)(128 / a);
    for (int T = 1; T <= Tmax; T = (T < 80 ? T + 1 : T * 2 + 1)) {
        const SplitPlan sp = split_plan(p, T, sms, k, act8);
        if (sp.s_gu < 1 || sp.s_gu > kMaxSplit || sp.s_dn < 1 || sp.s_dn > kMaxSplit)
            return fail_case("split count out of range", p, T, k, sms);
        if (sp.s_gu > 1 && (int)(d / kblk) / sp.s_gu < 8) return fail_case("gate/up range < 8 k-blocks", p, T, k, sms);
        if (sp.s_dn > 1 && (int)(std::min(F, Fs) / kblk) / sp.s_dn < 8)
            return fail_case("down range < 8 k-blocks", p, T, k, sms);
        const size_t Tt = T, Tv = Tt * k;
        // the partial planes run_layer addresses for this batch
        const size_t gu = sp.s_gu > 1 ? sp.s_gu * (Tv * 2 * F + Tt * 2 * Fs) : 0;
        const size_t dn = sp.s_dn * (Tv + Tt) * d;
        if (4 * std::max(gu, dn) > size_of(L.part)) return fail_case("partials too small", p, T, k, sms);
    }
    return true;
}

}  // namespace

int main() {
    std::mt19937 rng(7);
    const l4moe_dtype dts[] = {L4MOE_F32, L4MOE_BF16, L4MOE_FP8_E4M3, L4MOE_INT8};
    const int smss[] = {148, 132, 16, 2};
    int cases = 0;
    for (int c = 0; c < 4000; ++c) {
        l4moe_params p{};
        p.num_experts = (c % 7 == 0) ? 0 : 1 + (int)(rng() % 256);
        p.d_model = 64 * (1 + (int)(rng() % 96));
        p.shared_ffn = 64 * (1 + (int)(rng() % 160));
        p.expert_ffn = p.num_experts ? 64 * (1 + (int)(rng() % 160)) : 0;
        p.dtype = dts[rng() % 4];
        const int kmax = p.num_experts ? std::min(kMaxTopK, p.num_experts) : 1;
        const int k = 1 + (int)(rng() % kmax);
        const int Tmax = (c % 3 == 0) ? 1 + (int)(rng() % 100) : 1 + (int)(rng() % 20000);
        const bool act8 = p.dtype == L4MOE_FP8_E4M3 && (rng() & 1);
        if (!check(p, Tmax, k, smss[rng() % 4], act8)) return 1;
        ++cases;
    }
    // the workloads' own shapes at their token counts
    const int shapes[][4] = {{128, 4, 256, 256}, {5120, 16, 8192, 8192}, {5120, 128, 8192, 8192}, {5120, 0, 0, 16384}};
    for (auto& s : shapes)
        for (l4moe_dtype dt : dts)
            for (int Tmax : {1, 8, 32, 128, 4096, 8192, 16384}) {
                l4moe_params p{s[0], s[2], s[3], s[1], dt};
                if (!check(p, Tmax, 1, 148)) return 1;
                ++cases;
                if (dt == L4MOE_FP8_E4M3) {
                    if (!check(p, Tmax, 1, 148, true)) return 1;
                    ++cases;
                }
            }
    // the tensor-core router's shared memory, for every E it takes (E % 8 == 0,
    // up to 256; a launch's CTA takes all E experts, or 16 in the expert-split
    // form): its stages fit the limit it asks for, and the slice exchange
    // (128 token rows of n_pad + 4 floats) and the ranks' counts (4 rows of E
    // ints) fit its stage memory
    for (int E = 8; E <= 256; E += 8) {
        const int nst = rmma::stages(E);
        const size_t stage_mem = (size_t)nst * rmma::stage_bytes(E);
        const size_t recv = 4 * 128 * (size_t)(((E + 15) & ~15) + 4);
        if (nst < 4 || nst > rmma::MAX_STAGES || rmma::smem_bytes(E, nst) > rmma::SMEM_BYTES ||
            recv + 16 * (size_t)E > stage_mem || router_stage_cap(E) < 1) {
            printf("BAD router shared memory: E %d stages %d\n", E, nst);
            return 1;
        }
        ++cases;
    }
    // the workloads' top-1 bf16 routers at large batches finish the dispatch
    // themselves: every chunk's counts fit the last CTA's staging
    for (int E : {16, 128})
        for (int T : {17, 4096, 8192, 16384, 65536})
            if (router_max_chunks(T) > (size_t)router_stage_cap(E)) {
                printf("BAD router dispatch staging: E %d T %d chunks %zu cap %d\n", E, T, router_max_chunks(T),
                       router_stage_cap(E));
                return 1;
            }
    printf("OK %d\n", cases);
    return 0;
}
