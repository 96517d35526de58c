// Warp-specialised reverse-time adjoint scan (ParaGRU / ParaLSTM).
//
// The mathematics is that of adjoint.cuh: with mu_l = J_l^T lambda_l every
// step is the affine map mu_l = J_l^T mu_{l+1} + J_l^T g_l of the state
// entering it from later time (the transposed Newton system; page "ParaRNN:
// Apple destrava treino paralelo de RNNs não-lineares e escala pra 7B
// parâmetros", sections "A sacada: método de Newton" and "Engenharia pra
// escalar"), lambda_l = g_l + mu_{l+1}, du_l by the cell's chain rule, da as
// a deterministic sum.  The work of a CTA is split by role, as in the fused
// solve, so that no CTA-wide barrier sits inside the tile loop:
//   * CW compute warps, each owning two consecutive steps of a tile (tile =
//     2*CW steps x 128 channels, taken from the end of the sequence).  For
//     tile n a warp runs sweep 1 (Jacobians of its two steps, their
//     transposed maps folded), then sweep 2 of tile n-1 (its mu from the
//     tile's carry and its exclusive prefix; lambda, du and the da partial
//     of its steps).
//   * one control warp takes tickets, issues the TMA loads (gates, forward
//     states with the row before the tile, upstream gradients) into a ring,
//     turns the folds into exclusive prefixes (latest steps first), takes
//     the carry from the later tile's published value, and writes it.
// After sweep 2 the compute warps add their da partials of the tile in warp
// order (between two named barriers among them), so that da is reproducible.
#pragma once

#include <climits>

#include "adjoint.cuh"

namespace pararnn {

// NG: upstream gradient components staged per tile -- NS, or 1 when only the
// last component (h) has one (a ParaLSTM loss on h alone), which leaves room
// for more compute warps.
template <class Cell, class UT, int CW, int NG = Cell::NS>
struct AdjointWsLayout {
    static constexpr int G = Cell::G;
    static constexpr int NS = Cell::NS;
    static_assert(NG == NS || NG == 1, "staged upstream components");
    static constexpr int NC = Cell::Map::kFloats;
    static constexpr int Lc = 2 * CW;
    static constexpr int kStages = 3;
    static constexpr int kWork = 2;
    static constexpr size_t a128(size_t x) { return (x + 127) & ~size_t(127); }
    static constexpr size_t u_tx = size_t(Lc) * G * kDc * sizeof(UT);
    static constexpr size_t s_tx = size_t(Lc + 1) * kDc * 4;  // states from the row before the tile
    static constexpr size_t g_tx = size_t(Lc) * kDc * 4;
    // ring stage: gates | states [NS] | upstream [NG]
    static constexpr size_t off_u = 0;
    static constexpr size_t off_s = a128(u_tx);
    static constexpr size_t s_bytes = a128(s_tx);
    static constexpr size_t off_g = off_s + NS * s_bytes;
    static constexpr size_t g_bytes = a128(g_tx);
    static constexpr size_t stage_bytes = off_g + NG * g_bytes;
    // the upstream slot of component q (with NG = 1 only the last one is staged)
    static constexpr int g_slot(int q) { return NG == NS ? q : 0; }
    // work buffer: folds, then exclusive prefixes [NC][CW][kDc] | carry [NS][kDc]
    static constexpr size_t off_agg = 0;
    static constexpr size_t off_carry = a128(size_t(NC) * CW * kDc * 4);
    static constexpr size_t work_bytes = off_carry + a128(size_t(NS) * kDc * 4);
    static constexpr size_t off_work = kStages * stage_bytes;
    // the da partials of the compute warps [CW][G][kDc], one buffer: every
    // tile's are added up between two barriers of the compute warps
    static constexpr size_t off_dacc = off_work + kWork * work_bytes;
    static constexpr size_t off_misc = off_dacc + a128(size_t(CW) * G * kDc * 4);
    // misc: full, empty per stage; aggr, carry per work buffer; a job
    // (ticket, chunk, batch row, first channel) per stage; flags
    static constexpr size_t misc_bytes = a128((2 * kStages + 2 * kWork) * 8 + kStages * 16 + 8 * 4);
    static constexpr size_t smem_bytes = off_misc + misc_bytes;
    static constexpr int threads = 32 * (CW + 1);
    // descriptors hold inclusive values only: every look-back waits for them
    static constexpr int desc_words = TileDesc<typename Cell::Map, NS, false>::words;
    static constexpr bool fits = smem_bytes <= 232448;
};

// named barrier 1 over the compute warps only
template <int CW>
__device__ __forceinline__ void compute_sync_n()
{
    asm volatile("bar.sync 1, %0;" ::"n"(32 * CW) : "memory");
}

template <class Cell, class UT, int CW, int NG = Cell::NS>
__global__ void __launch_bounds__(32 * (CW + 1), 1)
    adjoint_ws_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_s0,
                      const __grid_constant__ CUtensorMap tm_s1, const __grid_constant__ CUtensorMap tm_g0,
                      const __grid_constant__ CUtensorMap tm_g1, const AdjointParams p)
{
    using LY = AdjointWsLayout<Cell, UT, CW, NG>;
    using Map = typename Cell::Map;
    using TD = TileDesc<Map, Cell::NS, false>;  // inclusive values only
    constexpr int G = LY::G, NS = LY::NS, NC = LY::NC, Lc = LY::Lc;
    // upstream gradient of component q present and staged (with NG = 1 the
    // host launches this kernel only when component 0 has none)
    auto staged = [&](int q) { return p.has_g[q] != 0 && (NG == NS || q == NS - 1); };
    constexpr int kStages = LY::kStages, kWork = LY::kWork;
    static_assert(LY::fits, "shared memory");

    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + LY::off_misc);  // [kStages]
    uint64_t* bar_empty = bar_full + kStages;                                // [kStages]
    uint64_t* bar_aggr = bar_empty + kStages;                                // [kWork]
    uint64_t* bar_carry = bar_aggr + kWork;                                  // [kWork]
    int4* s_job = reinterpret_cast<int4*>(bar_carry + kWork);                // [kStages]
    int* s_int = reinterpret_cast<int*>(s_job + kStages);                    // flags
    auto stage_at = [&](int i) { return smem + i * LY::stage_bytes; };
    auto work_at = [&](int i) { return smem + LY::off_work + i * LY::work_bytes; };
    auto compute_sync = [] { compute_sync_n<CW>(); };

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const bool ctl = (w == CW);
    WsHeader* hdr = p.hdr;
    int* err = &hdr->error;
    const long long D = p.D, L = p.L;
    const int BS = int(p.B) * p.S;

    if (tid == 0) {
        prefetch_tensormap(&tm_u);
        prefetch_tensormap(&tm_s0);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bar_full[i], 1);
            mbar_init(&bar_empty[i], CW);
        }
        for (int i = 0; i < kWork; ++i) {
            mbar_init(&bar_aggr[i], CW);
            mbar_init(&bar_carry[i], 1);
        }
        s_int[0] = 0;  // look-back failure seen by the control warp
        fence_mbar_init();
    }
    __syncthreads();

    if (ctl) {
        // ------------------------------------------------------ control warp
        auto issue = [&](int t, int stage) {  // lane 0 only
            if (error_raised(err) || s_int[0]) t = INT_MAX;
            if (t < p.n_tiles) {
                const int c = p.n_chunks - 1 - t / BS, rem = t - (t / BS) * BS;  // chunks from the end
                const int b = rem / p.S, d0 = (rem - b * p.S) * kDc;
                s_job[stage] = make_int4(t, c, b, d0);
                unsigned char* st = stage_at(stage);
                fence_proxy_async_shared();
                uint32_t bytes = uint32_t(LY::u_tx + NS * LY::s_tx);
#pragma unroll
                for (int q = 0; q < NS; ++q)
                    if (staged(q)) bytes += uint32_t(LY::g_tx);
                mbar_arrive_expect_tx(&bar_full[stage], bytes);
                tma_load_4d(st + LY::off_u, &tm_u, d0, 0, c * Lc, b, &bar_full[stage]);
                // rows c*Lc - 1 .. c*Lc + Lc - 1 (the row before the first chunk reads as zeros)
                tma_load_3d(st + LY::off_s, &tm_s0, d0, c * Lc - 1, b, &bar_full[stage]);
                if (NS == 2) tma_load_3d(st + LY::off_s + LY::s_bytes, &tm_s1, d0, c * Lc - 1, b, &bar_full[stage]);
                if (staged(0)) tma_load_3d(st + LY::off_g, &tm_g0, d0, c * Lc, b, &bar_full[stage]);
                if (NS == 2 && staged(1))
                    tma_load_3d(st + LY::off_g + LY::g_slot(1) * LY::g_bytes, &tm_g1, d0, c * Lc, b, &bar_full[stage]);
            } else {
                s_job[stage] = make_int4(INT_MAX, 0, 0, 0);
                mbar_arrive(&bar_full[stage]);
            }
            return t;
        };
        auto take = [&]() { return int(atomicAdd(&hdr->tick[0], 1u)); };
        int tk[kStages];
        if (lane == 0) {
#pragma unroll
            for (int i = 0; i < kStages; ++i) tk[i] = issue(take(), i);
        }
#pragma unroll
        for (int i = 0; i < kStages; ++i) tk[i] = __shfl_sync(0xffffffffu, tk[i], 0);
        for (int n = 0;; ++n) {
            const int s = n % kStages, wb = n % kWork;
            int ticket = tk[0];
#pragma unroll
            for (int i = 1; i < kStages; ++i)
                if (s == i) ticket = tk[i];
            if (ticket < p.n_tiles) {
                const int c = p.n_chunks - 1 - ticket / BS;
                bool ok = mbar_wait_bounded(&bar_aggr[wb], uint32_t(n / kWork) & 1u, err, p.wait_ns);
                LookbackProbe<Map, NS> pr;
                const bool has_pred = c < p.n_chunks - 1;  // a later chunk exists
                if (has_pred) lookback_probe<Map, NS, false, TD>(pr, ticket - BS, p.desc, lane);
                // folds -> exclusive prefixes in place, latest segment first;
                // their composition is the tile's map
                float* agg = reinterpret_cast<float*>(work_at(wb) + LY::off_agg);
                Map run[kV];
#pragma unroll
                for (int j = 0; j < kV; ++j) run[j] = Map::identity();
                for (int seg = CW - 1; seg >= 0; --seg) {
                    Map m[kV];
#pragma unroll
                    for (int i = 0; i < NC; ++i) {
                        float* row = agg + (i * CW + seg) * kDc + lane * kV;
                        F4 v = load4(row);
                        float v4[kV];
#pragma unroll
                        for (int j = 0; j < kV; ++j) {
                            m[j].set(i, v.v[j]);
                            v4[j] = run[j].get(i);
                        }
                        store4(row, v4);
                    }
#pragma unroll
                    for (int j = 0; j < kV; ++j) run[j] = compose(m[j], run[j]);
                }
                // the carry is the later tile's inclusive value (waited for,
                // never assembled from aggregates, so that every run adds in
                // the same order); mu_{L+1} = 0 enters the last chunk
                float y[NS][kV];
#pragma unroll
                for (int q = 0; q < NS; ++q)
#pragma unroll
                    for (int j = 0; j < kV; ++j) y[q][j] = 0.f;
                if (has_pred)
                    ok = lookback_resolve<Map, NS, false, TD>(ticket, BS, 0, y, p.desc, lane, err, p.wait_ns, pr) && ok;
                if (__all_sync(0xffffffffu, ok)) {
                    float incl[NS][kV];
#pragma unroll
                    for (int j = 0; j < kV; ++j) {
                        float x[NS], z[NS];
#pragma unroll
                        for (int q = 0; q < NS; ++q) x[q] = y[q][j];
                        apply(run[j], x, z);
#pragma unroll
                        for (int q = 0; q < NS; ++q) incl[q][j] = z[q];
                    }
                    publish_inclusive<Map, NS, TD>(p.desc, ticket, 0, incl, lane);
                }
                float* car = reinterpret_cast<float*>(work_at(wb) + LY::off_carry);
#pragma unroll
                for (int q = 0; q < NS; ++q) store4(car + q * kDc + lane * kV, y[q]);
                if (!__all_sync(0xffffffffu, ok) && lane == 0) s_int[0] = 1;
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_carry[wb]);
            }
            if (ticket >= p.n_tiles) break;
            // refill the stage released by the tile before this one
            if (n >= 1) {
                const int sp = (n - 1) % kStages;
                int t = 0;
                if (lane == 0) {
                    (void)mbar_wait_bounded(&bar_empty[sp], uint32_t((n - 1) / kStages) & 1u, err, p.wait_ns);
                    t = issue(take(), sp);
                }
                t = __shfl_sync(0xffffffffu, t, 0);
#pragma unroll
                for (int i = 0; i < kStages; ++i)
                    if (sp == i) tk[i] = t;
            }
        }
    } else {
        // ------------------------------------------------------ compute warps
        const int ra = 2 * w, rb = 2 * w + 1;  // this warp's steps in the tile (rb is the later)
        int4 prev = make_int4(INT_MAX, 0, 0, 0);
        for (int n = 0;; ++n) {
            const int s = n % kStages, wb = n % kWork;
            (void)mbar_wait_bounded(&bar_full[s], uint32_t(n / kStages) & 1u, err, p.wait_ns);
            const int4 job = s_job[s];
            const bool valid = job.x < p.n_tiles;
            // state before step `row`, upstream gradient at `row`, gates of `row`
            auto step_inputs = [&](const unsigned char* st, int row, int c, int b, int dch, bool chv,
                                   float (&sv)[NS][kV], float (&gv)[NS][kV], F4 (&ug)[G]) {
                const float* ss = reinterpret_cast<const float*>(st + LY::off_s);
                const float* sg = reinterpret_cast<const float*>(st + LY::off_g);
                const UT* su = reinterpret_cast<const UT*>(st + LY::off_u);
#pragma unroll
                for (int q = 0; q < NS; ++q) {
                    F4 x = load4(ss + q * (LY::s_bytes / 4) + row * kDc + lane * kV);  // row-1 of the chunk, shifted by one
                    if (row == 0 && c == 0) {
                        x = F4{{0.f, 0.f, 0.f, 0.f}};
                        if (chv && p.s0[q]) x = load4(p.s0[q] + b * D + dch);
                    }
                    F4 z{{0.f, 0.f, 0.f, 0.f}};
                    if (staged(q)) z = load4(sg + LY::g_slot(q) * (LY::g_bytes / 4) + row * kDc + lane * kV);
#pragma unroll
                    for (int j = 0; j < kV; ++j) {
                        sv[q][j] = x.v[j];
                        gv[q][j] = z.v[j];
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) ug[g] = load4(su + (row * G + g) * kDc + lane * kV);
            };
            float wv[G][kV];
            if (valid) {
                // ---- sweep 1 of tile n: the transposed maps of steps rb, ra folded
                const unsigned char* st = stage_at(s);
                const int c = job.y, b = job.z, d0 = job.w;
                const int dch = d0 + lane * kV;
                const bool chv = dch < D;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    F4 x = chv ? load4(p.a + g * D + dch) : F4{{0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                    for (int j = 0; j < kV; ++j) wv[g][j] = x.v[j];
                }
                Map agg[kV];
#pragma unroll
                for (int j = 0; j < kV; ++j) agg[j] = Map::identity();
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int row = k == 0 ? rb : ra;
                    float sv[NS][kV], gv[NS][kV];
                    F4 ug[G];
                    step_inputs(st, row, c, b, dch, chv, sv, gv, ug);
#pragma unroll
                    for (int j = 0; j < kV; ++j) {
                        float s1[NS], uu[G], aa[G], f[NS], g1[NS];
#pragma unroll
                        for (int q = 0; q < NS; ++q) {
                            s1[q] = sv[q][j];
                            g1[q] = gv[q][j];
                        }
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            uu[g] = ug[g].v[j];
                            aa[g] = wv[g][j];
                        }
                        Map J;
                        Cell::eval(s1, uu, aa, f, J);
                        agg[j] = compose(transpose_map(J, g1), agg[j]);
                    }
                }
                float* sagg = reinterpret_cast<float*>(work_at(wb) + LY::off_agg);
#pragma unroll
                for (int i = 0; i < NC; ++i) {
                    float v4[kV];
#pragma unroll
                    for (int j = 0; j < kV; ++j) v4[j] = agg[j].get(i);
                    store4(sagg + (i * CW + w) * kDc + lane * kV, v4);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_aggr[wb]);
            }
            if (prev.x < p.n_tiles) {
                // ---- sweep 2 of tile n-1: lambda, du, da partial, mu
                const int sp_ = (n - 1) % kStages, wp = (n - 1) % kWork;
                (void)mbar_wait_bounded(&bar_carry[wp], uint32_t((n - 1) / kWork) & 1u, err, p.wait_ns);
                const unsigned char* st = stage_at(sp_);
                const unsigned char* wk = work_at(wp);
                const int c = prev.y, b = prev.z, d0 = prev.w;
                const long long l0 = (long long)c * Lc;
                const int dch = d0 + lane * kV;
                const bool chv = dch < D && !s_int[0];
                float av[G][kV];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    F4 x = dch < D ? load4(p.a + g * D + dch) : F4{{0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                    for (int j = 0; j < kV; ++j) av[g][j] = x.v[j];
                }
                // mu entering this warp's steps from later time
                float mu[NS][kV];
                {
                    const float* spre = reinterpret_cast<const float*>(wk + LY::off_agg);
                    const float* car = reinterpret_cast<const float*>(wk + LY::off_carry);
                    Map pre[kV];
#pragma unroll
                    for (int i = 0; i < NC; ++i) {
                        F4 v = load4(spre + (i * CW + w) * kDc + lane * kV);
#pragma unroll
                        for (int j = 0; j < kV; ++j) pre[j].set(i, v.v[j]);
                    }
#pragma unroll
                    for (int j = 0; j < kV; ++j) {
                        float x[NS], y[NS];
#pragma unroll
                        for (int q = 0; q < NS; ++q) x[q] = car[q * kDc + lane * kV + j];
                        apply(pre[j], x, y);
#pragma unroll
                        for (int q = 0; q < NS; ++q) mu[q][j] = y[q];
                    }
                }
                float dacc[G][kV];
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int j = 0; j < kV; ++j) dacc[g][j] = 0.f;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int row = k == 0 ? rb : ra;
                    const long long l = l0 + row;
                    const bool lv = l < L;
                    float sv[NS][kV], gv[NS][kV];
                    F4 ug[G];
                    step_inputs(st, row, c, b, dch, dch < D, sv, gv, ug);
                    float duv[G][kV];
#pragma unroll
                    for (int j = 0; j < kV; ++j) {
                        float s1[NS], uu[G], aa[G], lam[NS], d1[G], da1[G], m1[NS];
#pragma unroll
                        for (int q = 0; q < NS; ++q) {
                            s1[q] = sv[q][j];
                            lam[q] = gv[q][j] + mu[q][j];
                        }
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            uu[g] = ug[g].v[j];
                            aa[g] = av[g][j];
                            da1[g] = 0.f;
                        }
                        Cell::vjp(s1, uu, aa, lam, d1, da1, m1);
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            duv[g][j] = d1[g];
                            if (lv) dacc[g][j] += da1[g];
                        }
#pragma unroll
                        for (int q = 0; q < NS; ++q) mu[q][j] = m1[q];
                    }
                    if (lv && chv) {
#pragma unroll
                        for (int g = 0; g < G; ++g) __stcg(reinterpret_cast<float4*>(p.du + (((b * L + l) * G + g) * D + dch)),
                                                           make_float4(duv[g][0], duv[g][1], duv[g][2], duv[g][3]));
                    }
                    if (l == 0 && chv) {
#pragma unroll
                        for (int q = 0; q < NS; ++q)
                            if (p.ds0[q]) store4(p.ds0[q] + b * D + dch, mu[q]);
                    }
                }
                // the tile's da partial: every warp's sums in shared memory,
                // then each warp adds up a slice of them in warp order
                float* sd = reinterpret_cast<float*>(smem + LY::off_dacc);
#pragma unroll
                for (int g = 0; g < G; ++g) store4(sd + (w * G + g) * kDc + lane * kV, dacc[g]);
                compute_sync();
                if (lane == 0) mbar_arrive(&bar_empty[sp_]);
                float* part = p.partial + (((size_t)b * p.n_chunks + c) * p.S + d0 / kDc) * G * kDc;
                for (int i = w * 32 + lane; i < G * kDc; i += 32 * CW) {
                    float acc = 0.f;
                    for (int ww = 0; ww < CW; ++ww) acc += sd[ww * G * kDc + i];
                    part[i] = acc;
                }
                compute_sync();  // the buffer is free for the next tile's partials
            }
            if (!valid) break;
            prev = job;
        }
    }
}

}  // namespace pararnn
