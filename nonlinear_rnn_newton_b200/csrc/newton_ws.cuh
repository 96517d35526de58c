// Warp-specialised fused Newton solve (ParaGRU / ParaLSTM).
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros" -- "A sacada: método de Newton" (each iteration linearises
// every step and solves the linear SSM delta_l = J_l delta_{l-1} - F_l with a
// parallel scan), "Engenharia pra escalar" (diagonal / 2x2 Jacobians; Newton
// iterations, system assembly and the parallel reduction fused in one kernel).
//
// The mathematics is that of newton.cuh (direct form of the Newton step
// s^{k+1}_l = J_l s^{k+1}_{l-1} + o_l with o_l = f_l - J_l s^k_{l-1}; residual
// of the updated states for the convergence test; grid barrier and a common
// decision between iterations).  The work of a CTA is split by role so that
// no CTA-wide barrier sits inside the tile loop:
//   * CW compute warps, each owning two consecutive steps of a tile
//     (tile = 2*CW steps x 128 channels).  For tile n a warp runs sweep 1
//     (cell, Jacobian and offsets of its two steps, evaluated together so
//     they share reciprocals; fold of its two maps), then sweep 2 of tile n-1
//     (state entering its steps = its prefix map applied to the tile's carry;
//     the new states; residual of the new states).  The Jacobians of the
//     previous tile wait in registers, the offsets in shared memory.
//   * one control warp takes tickets (each worth a group of consecutive chunks
//     of one sequence) and issues the TMA loads (gates, previous states, the
//     slab's recurrence weights and the state entering the chunk from the
//     last pass) into a four-stage ring; for tile n it starts the look-back's
//     first read, turns the compute warps' folds into exclusive prefixes in
//     place (their composition is the tile's aggregate), finishes the
//     decoupled look-back against other CTAs -- or, inside a group, takes the
//     inclusive value of the tile before -- and writes the tile's carry.
// A tile's gates and states live in a ring stage from their load until its
// sweep 2; the folds, offsets and carry live in one of two work buffers.
// Hand-offs use mbarriers (full: loads landed; aggr: folds written; carry:
// prefixes and carry written; empty: stage released).  Every wait is bounded.
#pragma once

#include <climits>

#include "newton.cuh"

namespace pararnn {

#ifndef PARARNN_WS_STAGES
#define PARARNN_WS_STAGES 4
#endif
constexpr int kStages = PARARNN_WS_STAGES;  // TMA ring
constexpr int kWork = 2;    // per-tile work buffers (tiles n-1 and n are live)
// A ticket hands out a group of kGroup = 2 consecutive chunks of one
// sequence; they run back to back in one CTA.  The decoupled look-back works
// on groups: the group's aggregate (the composition of its two tiles' maps)
// and its inclusive value (the state leaving it) are published in one
// descriptor per group, numbered like the tickets (group chunk * B * S +
// sequence), so a look-back steps back one group per read and never waits on
// a tile that publishes nothing.  The second tile takes its carry from the
// first in registers.  (Longer groups would need the control warp to wait
// for folds the compute warps can only produce after the first tile's carry,
// so two is the longest that can be prepared ahead.)
constexpr int kGroup = 2;

// Look-back descriptors a solve uses: one per group of every sequence.
__host__ __device__ constexpr long long solve_desc_count(int n_chunks, long long BS)
{
    return (long long)((n_chunks + kGroup - 1) / kGroup) * BS;
}


// CW: compute warps = row pairs (two steps each) in a tile.
template <class Cell, class UT, int CW>
struct NewtonWsLayout {
    static constexpr int G = Cell::G;
    static constexpr int NS = Cell::NS;
    static constexpr int NC = Cell::Map::kFloats;
    static constexpr int Lc = 2 * CW;  // two steps per compute warp
    static constexpr size_t a128(size_t x) { return (x + 127) & ~size_t(127); }
    // bytes one load of each kind delivers
    static constexpr size_t u_tx = size_t(Lc) * G * kDc * sizeof(UT);  // gate tile
    static constexpr size_t s_tx = size_t(Lc) * kDc * 4;                // state tile, one component
    static constexpr size_t a_tx = size_t(G) * kDc * 4;                 // recurrence weights of the slab
    static constexpr size_t bnd_tx = size_t(kDc) * 4;                   // boundary row, one component
    // ring stage: gates | states [NS] | weights | boundary [NS]
    static constexpr size_t off_u = 0;
    static constexpr size_t off_s = off_u + a128(u_tx);
    static constexpr size_t s_bytes = a128(s_tx);
    static constexpr size_t off_a = off_s + NS * s_bytes;
    static constexpr size_t off_bnd = off_a + a128(a_tx);
    static constexpr size_t stage_bytes = off_bnd + a128(NS * bnd_tx);
    // work buffer: folds, then exclusive prefixes [NC][CW][kDc] | offsets of
    // each warp's second step [NS][CW][kDc] | tile carry [NS][kDc]
    static constexpr size_t off_agg = 0;
    static constexpr size_t off_last = off_agg + a128(size_t(NC) * CW * kDc * 4);
    static constexpr size_t off_carry = off_last + a128(size_t(NS) * CW * kDc * 4);
    static constexpr size_t work_bytes = off_carry + a128(size_t(NS) * kDc * 4);
    static constexpr size_t off_work = kStages * stage_bytes;
    static constexpr size_t off_misc = off_work + kWork * work_bytes;
    // misc: barriers (full, empty per stage; aggr, carry per work buffer), a
    // job (ticket, chunk, batch row, first channel) per stage, 8 flags,
    // 2*(CW+1) residual slots
    static constexpr int CWT = CW;  // compute warps
    static constexpr size_t misc_bytes =
        a128((2 * kStages + 2 * kWork) * 8 + kStages * 16 + 8 * 4 + 2 * (CWT + 1) * 4);
    static constexpr size_t smem_bytes = off_misc + misc_bytes;
    static constexpr int threads = 32 * (CWT + 1);
    static constexpr bool fits = smem_bytes <= 232448;  // opt-in shared memory per CTA
};

// Whether passes that continue may leave residuals out (see sweep 2): the
// one-component cells; a two-component cell's own specialisation may opt in
// (the built-in ParaLSTM measured no faster with it).
template <class Cell>
struct PartialResiduals {
    static constexpr bool value = Cell::NS == 1;
};

// both halves finite (NaN and inf fail the comparison)
__device__ __forceinline__ bool finite2(float2 v)
{
    return fabsf(v.x) <= 3.40282347e38f && fabsf(v.y) <= 3.40282347e38f;
}

// Seg: the segment-pass form (warm start and a separate linearisation point
// for chunk 0, read from the workspace header); a template parameter so that
// the plain solve keeps its own code.
template <class Cell, class UT, int CW, bool Seg = false, int LB = 2>
__global__ void __launch_bounds__(32 * (CW + 1), 1)
    newton_solve_ws_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_s0,
                           const __grid_constant__ CUtensorMap tm_s1, const __grid_constant__ CUtensorMap tm_a,
                           const __grid_constant__ CUtensorMap tm_bnd, const NewtonParams p)
{
    using LY = NewtonWsLayout<Cell, UT, CW>;
    using Map = typename Cell::Map;
    using Packed = typename Cell::Packed;
    using Rows2 = typename Packed::Rows2;
    using Map2 = typename Packed::Map2;
    using Jac2 = typename Packed::Jac2;
    constexpr int G = LY::G, NS = LY::NS, NC = LY::NC, Lc = LY::Lc, CWT = LY::CWT;
    constexpr int CV = kV, NP = kV / 2;  // channels and channel pairs of a compute lane
    // look-backs step back over aggregates (LB = 1), wait for inclusive
    // values (LB = 0), or follow p.lb_walk (LB = 2)
    const bool walk = LB == 2 ? p.lb_walk != 0 : LB == 1;
    // descriptors: inclusive values only when no look-back steps back
    using TD = TileDesc<Map, NS, LB != 0>;
    static_assert(LY::fits, "shared memory");

    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + LY::off_misc);  // [kStages]
    uint64_t* bar_empty = bar_full + kStages;                                // [kStages]
    uint64_t* bar_aggr = bar_empty + kStages;                                // [kWork]
    uint64_t* bar_carry = bar_aggr + kWork;                                  // [kWork]
    int4* s_job = reinterpret_cast<int4*>(bar_carry + kWork);                // [kStages]
    int* s_int = reinterpret_cast<int*>(s_job + kStages);                    // misc flags
    float* s_red = reinterpret_cast<float*>(s_int + 8);                      // [2 * (CWT + 1)]
    auto stage_at = [&](int i) { return smem + i * LY::stage_bytes; };
    auto work_at = [&](int i) { return smem + LY::off_work + i * LY::work_bytes; };

    const int tid = threadIdx.x;
    const int w = tid >> 5;
    const int lane = tid & 31;
    const bool ctl = (w == CWT);
    WsHeader* hdr = p.hdr;
    int* err = &hdr->error;
    const long long D = p.D, L = p.L;
    const int BS = int(p.B) * p.S;
    const int Dpad = p.S * kDc;

    if (tid == 0) {
        prefetch_tensormap(&tm_u);
        prefetch_tensormap(&tm_s0);
        if (NS == 2) prefetch_tensormap(&tm_s1);
        prefetch_tensormap(&tm_a);
        prefetch_tensormap(&tm_bnd);
    }

    // pass 0 may have run already, fused with the input projection: then the
    // decision after it comes first (from the residuals that kernel left)
    const int k0 = hdr->k0;
    if (tid == 0 && blockIdx.x == 0) hdr->t_pass[k0] = global_timer_ns();
    if (k0 == 1) {
        if (tid == 0) {
            NewtonDecision d = newton_decide(hdr, 0, 0, true, p.tol, p.max_iters);
            if (!d.cont && blockIdx.x == 0) newton_publish(hdr, d, 0);
            s_int[2] = d.cont;
            s_int[3] = d.zero;
        }
        __syncthreads();
        if (!s_int[2]) {
            if (s_int[3]) newton_zero_states<NS>(p, tid, blockDim.x);
            return;
        }
    }

    for (int k = k0;; ++k) {
        const int slot = k % 3;
        const bool first = (k == 0) && !(Seg && hdr->seg_warm);  // the pass starts from H^0 = 0
        if (tid == 0) {
            if (blockIdx.x == 0) {
                // slot (k+1)%3 was last used two passes ago; every CTA is past it
                hdr->tick[(k + 1) % 3] = 0u;
                hdr->res[(k + 1) % 3] = 0u;
                hdr->over[(k + 1) % 3] = 0u;
            }
            // fresh barriers every pass (no copy is in flight between passes)
            for (int i = 0; i < kStages; ++i) {
                if (k > k0) {
                    mbar_inval(&bar_full[i]);
                    mbar_inval(&bar_empty[i]);
                }
                mbar_init(&bar_full[i], 1);
                mbar_init(&bar_empty[i], CWT);
            }
            for (int i = 0; i < kWork; ++i) {
                if (k > k0) {
                    mbar_inval(&bar_aggr[i]);
                    mbar_inval(&bar_carry[i]);
                }
                mbar_init(&bar_aggr[i], CWT);
                mbar_init(&bar_carry[i], 1);
            }
            s_int[0] = 0;  // look-back failure seen by the control warp
            fence_mbar_init();
        }
        __syncthreads();
        float rpost = 0.f, rpre = 0.f;  // max |F|, NaN kept

        if (ctl) {
            // ------------------------------------------------ control warp
            auto issue = [&](int t, int stage) {  // lane 0 only
                if (error_raised(err) || s_int[0]) t = INT_MAX;
                if (t < p.n_tiles) {
                    const int c = t / BS, rem = t - (t / BS) * BS;
                    const int b = rem / p.S, d0 = (rem - b * p.S) * kDc;
                    s_job[stage] = make_int4(t, c, b, d0);
                    unsigned char* st = stage_at(stage);
                    fence_proxy_async_shared();
                    const bool with_bnd = !first && c > 0;  // state entering the chunk, from the last pass
                    const uint32_t bytes = uint32_t(LY::u_tx + LY::a_tx + (first ? 0 : NS * LY::s_tx) +
                                                    (with_bnd ? NS * LY::bnd_tx : 0));
                    mbar_arrive_expect_tx(&bar_full[stage], bytes);
                    tma_load_4d(st + LY::off_u, &tm_u, d0, 0, c * Lc, b, &bar_full[stage]);
                    tma_load_2d(st + LY::off_a, &tm_a, d0, 0, &bar_full[stage]);
                    if (!first) {
                        tma_load_3d(st + LY::off_s, &tm_s0, d0, c * Lc, b, &bar_full[stage]);
                        if (NS == 2)
                            tma_load_3d(st + LY::off_s + LY::s_bytes, &tm_s1, d0, c * Lc, b, &bar_full[stage]);
                    }
                    if (with_bnd) {
#pragma unroll
                        for (int q = 0; q < NS; ++q)
                            tma_load_3d(st + LY::off_bnd + q * LY::bnd_tx, &tm_bnd, d0, c - 1,
                                        ((k & 1) * NS + q) * int(p.B) + b, &bar_full[stage]);
                    }
                } else {
                    s_job[stage] = make_int4(INT_MAX, 0, 0, 0);
                    mbar_arrive(&bar_full[stage]);
                }
                return t;
            };
            // the next tile: the rest of the current group, then a new group
            // ticket (lane 0 only; tickets count groups, tiles are numbered
            // chunk * BS + sequence)
            const int n_groups = ((p.n_chunks + kGroup - 1) / kGroup) * BS;
            int g_c = 0, g_end = 0, g_q = 0;  // next chunk, end chunk and sequence of the group
            auto next_tile = [&]() {
                if (g_c >= g_end) {
                    const int gt = int(atomicAdd(&hdr->tick[slot], 1u));
                    if (gt >= n_groups) return INT_MAX;
                    g_q = gt % BS;
                    g_c = (gt / BS) * kGroup;
                    g_end = min(g_c + kGroup, p.n_chunks);
                }
                return (g_c++) * BS + g_q;
            };
            // tickets of the tiles in the ring, by stage
            int tk[kStages];
            if (lane == 0) {
#pragma unroll
                for (int i = 0; i < kStages; ++i) tk[i] = issue(next_tile(), i);
            }
#pragma unroll
            for (int i = 0; i < kStages; ++i) tk[i] = __shfl_sync(0xffffffffu, tk[i], 0);
            float y_inc[NS][kV];  // inclusive value of the last tile handled here
            // folds of work buffer `wkb` -> exclusive prefixes (in place); returns
            // the tile's aggregate (the last inclusive prefix) in `run`
            auto prefix = [&](int wkb, Map (&run)[kV]) {
                float* agg = reinterpret_cast<float*>(work_at(wkb) + LY::off_agg);
#pragma unroll
                for (int j = 0; j < kV; ++j) run[j] = Map::identity();
                for (int seg = 0; seg < CW; ++seg) {
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
            };
            // A group's second tile is prepared while its first tile's look-back
            // read is in flight: its prefixes are computed (run_pre) before the
            // look-back resolves, so that the group's aggregate can be
            // published first, and its carry follows from the first tile's.
            bool pre_done = false;  // the next tile's prefixes are computed (run_pre)
            Map run_pre[kV];
            for (int n = 0;; ++n) {
                const int s = n % kStages, wb = n % kWork;
                int ticket = tk[0];
#pragma unroll
                for (int i = 1; i < kStages; ++i)
                    if (s == i) ticket = tk[i];
                if (ticket >= p.n_tiles) break;
                const int c = ticket / BS, rem = ticket - (ticket / BS) * BS;
                const int b = rem / p.S, d0 = (rem - b * p.S) * kDc;
                const int dch = d0 + lane * kV;
                // inside a group the tile before ran here: its inclusive value
                // (y_inc) is this tile's carry
                const bool local = (c % kGroup) != 0;
                const int gt = (c / kGroup) * BS + rem;  // group ticket (descriptor index)
                LookbackProbe<Map, NS> pr;
                float* car = reinterpret_cast<float*>(work_at(wb) + LY::off_carry);
                bool ok = true;
                Map run[kV];
                if (local && pre_done) {
#pragma unroll
                    for (int j = 0; j < kV; ++j) run[j] = run_pre[j];
                } else {
                    ok = mbar_wait_bounded(&bar_aggr[wb], uint32_t(n / kWork) & 1u, err, p.wait_ns);
                    // first look-back read, in flight while the folds are composed
                    // (issued only now, so that it sees predecessors as late as possible)
                    if (c > 0 && !local) {
                        if (walk) lookback_probe<Map, NS, LB != 0, TD>(pr, gt - BS, p.desc, lane);
                        else lookback_probe<Map, NS, false, TD>(pr, gt - BS, p.desc, lane);
                    }
                    prefix(wb, run);
                }
                float y[NS][kV];
                // waiting for inclusive values needs none of this group's
                // maps: a group's first carry then goes out before the second
                // tile's folds are composed
                const bool early = !walk && !local;
                if (local) {
                    // carry = inclusive value of the group's previous tile
#pragma unroll
                    for (int q = 0; q < NS; ++q)
#pragma unroll
                        for (int j = 0; j < kV; ++j) y[q][j] = y_inc[q][j];
                    pre_done = false;
                } else {
                    if (early) {
                        if (c > 0) {
                            ok = lookback_resolve<Map, NS, false, TD>(gt, BS, k, y, p.desc, lane, err, p.wait_ns, pr) &&
                                 ok;
                        } else {
#pragma unroll
                            for (int q = 0; q < NS; ++q) {
                                F4 x{{0.f, 0.f, 0.f, 0.f}};
                                if (dch < D && p.s0[q]) x = load4(p.s0[q] + b * D + dch);
#pragma unroll
                                for (int j = 0; j < kV; ++j) y[q][j] = x.v[j];
                            }
                        }
#pragma unroll
                        for (int q = 0; q < NS; ++q) store4(car + q * kDc + lane * kV, y[q]);
                        if (!__all_sync(0xffffffffu, ok) && lane == 0) s_int[0] = 1;
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bar_carry[wb]);
                    }
                    // the group's second tile (the next in the ring): its
                    // prefixes now, while the look-back read is in flight
                    bool two = false;
                    if (c + 1 < p.n_chunks) {
                        const int n1 = n + 1, s1 = n1 % kStages;
                        int t1 = tk[0];
#pragma unroll
                        for (int i = 1; i < kStages; ++i)
                            if (s1 == i) t1 = tk[i];
                        if (t1 == ticket + BS) {
                            ok = mbar_wait_bounded(&bar_aggr[n1 % kWork], uint32_t(n1 / kWork) & 1u, err, p.wait_ns) &&
                                 ok;
                            prefix(n1 % kWork, run_pre);
                            pre_done = two = true;
                        } else {
                            ok = false;  // the group's tiles are always issued back to back
                        }
                    }
                    if (!early) {
                        if (c > 0) {
                            // stepping back: the group's aggregate (both
                            // tiles' maps composed) goes out first, for
                            // look-backs that step over it
                            Map gagg[kV];
#pragma unroll
                            for (int j = 0; j < kV; ++j) gagg[j] = two ? compose(run_pre[j], run[j]) : run[j];
                            if constexpr (LB != 0) {  // (with LB = 0 every head carry goes out early)
                                publish_aggregate<Map, NS, TD>(p.desc, gt, k, gagg, lane);
                                ok = lookback_resolve<Map, NS, true, TD>(gt, BS, k, y, p.desc, lane, err, p.wait_ns,
                                                                         pr) &&
                                     ok;
                            }
                        } else {
                            // the sequence's first group: the initial state
#pragma unroll
                            for (int q = 0; q < NS; ++q) {
                                F4 x{{0.f, 0.f, 0.f, 0.f}};
                                if (dch < D && p.s0[q]) x = load4(p.s0[q] + b * D + dch);
#pragma unroll
                                for (int j = 0; j < kV; ++j) y[q][j] = x.v[j];
                            }
                        }
                    }
                }
                // the state leaving this tile; at a group's head, also the
                // state leaving the group (its inclusive value)
#pragma unroll
                for (int j = 0; j < kV; ++j) {
                    float x[NS], z[NS];
#pragma unroll
                    for (int q = 0; q < NS; ++q) x[q] = y[q][j];
                    apply(run[j], x, z);
#pragma unroll
                    for (int q = 0; q < NS; ++q) y_inc[q][j] = z[q];
                }
                if (!local && __all_sync(0xffffffffu, ok)) {
                    float incl[NS][kV];
#pragma unroll
                    for (int j = 0; j < kV; ++j) {
                        float x[NS], z[NS];
#pragma unroll
                        for (int q = 0; q < NS; ++q) x[q] = y_inc[q][j];
                        if (pre_done) apply(run_pre[j], x, z);
#pragma unroll
                        for (int q = 0; q < NS; ++q) incl[q][j] = pre_done ? z[q] : x[q];
                    }
                    publish_inclusive<Map, NS, TD>(p.desc, gt, k, incl, lane);
                }
                if (!early) {
#pragma unroll
                    for (int q = 0; q < NS; ++q) store4(car + q * kDc + lane * kV, y[q]);
                }
                if (!__all_sync(0xffffffffu, ok) && lane == 0) s_int[0] = 1;
                __syncwarp();
                if (!early && lane == 0) mbar_arrive(&bar_carry[wb]);
                // refill the stage released by the tile before this one
                if (n >= 1) {
                    const int sp = (n - 1) % kStages;
                    int t = 0;
                    if (lane == 0) {
                        (void)mbar_wait_bounded(&bar_empty[sp], uint32_t((n - 1) / kStages) & 1u, err, p.wait_ns);
                        t = issue(next_tile(), sp);
                    }
                    t = __shfl_sync(0xffffffffu, t, 0);
#pragma unroll
                    for (int i = 0; i < kStages; ++i)
                        if (sp == i) tk[i] = t;
                }
            }
        } else {
            // ------------------------------------------------ compute warps
            const int rp = w;             // this warp's row pair
            const int cofs = lane * CV;   // first channel of this lane in the tile
            const int ra = 2 * rp, rb = 2 * rp + 1;  // this warp's two steps in the tile
            int4 prev = make_int4(INT_MAX, 0, 0, 0);  // job of the previous tile
            Jac2 Jp[2][NP];  // Jacobians of the previous tile's two steps (per pair)
            for (int n = 0;; ++n) {
                const int s = n % kStages, wb = n % kWork;
                (void)mbar_wait_bounded(&bar_full[s], uint32_t(n / kStages) & 1u, err, p.wait_ns);
                const int4 job = s_job[s];
                const bool valid = job.x < p.n_tiles;
                // whether a tile of this pass has found a residual above tol
                // (read now, used in sweep 2 below: the load is in flight
                // during sweep 1)
                // (never set where p.skip_res is 0)
                const int over_seen = (PartialResiduals<Cell>::value && lane == 0)
                                          ? ld_relaxed_gpu(reinterpret_cast<const int*>(&hdr->over[slot]))
                                          : 0;
                Jac2 Jn[2][NP];
                if (valid) {
                    // ---- sweep 1 of tile n
                    unsigned char* st = stage_at(s);
                    unsigned char* wk = work_at(wb);
                    const UT* su = reinterpret_cast<const UT*>(st + LY::off_u);
                    float* ss = reinterpret_cast<float*>(st + LY::off_s);
                    const float* sa = reinterpret_cast<const float*>(st + LY::off_a);
                    const float* sbnd = reinterpret_cast<const float*>(st + LY::off_bnd);
                    float* slast = reinterpret_cast<float*>(wk + LY::off_last);
                    float* sagg = reinterpret_cast<float*>(wk + LY::off_agg);
                    const int c = job.y, b = job.z, d0 = job.w;
                    const int l0 = c * Lc;
                    const int dch = d0 + cofs;
                    const bool chv = dch < D;
                    float2 wv[G][NP];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        FV<CV> x = loadv<CV>(sa + g * kDc + cofs);  // zero beyond D (TMA fill)
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) wv[g][jp] = make_float2(x.v[2 * jp], x.v[2 * jp + 1]);
                    }
                    // s^k before step a, s^k at steps a and b
                    float2 sp[NS][NP], ska[NS][NP], skb[NS][NP];
#pragma unroll
                    for (int q = 0; q < NS; ++q) {
                        FV<CV> x, xa, xb;
#pragma unroll
                        for (int j = 0; j < CV; ++j) x.v[j] = xa.v[j] = xb.v[j] = 0.f;
                        if (rp == 0) {
                            if (c == 0) {
                                const float* lin = p.s0[q];
                                if (Seg && hdr->seg_lin[q]) lin = reinterpret_cast<const float*>(hdr->seg_lin[q]);
                                if (chv && lin) x = loadv<CV>(lin + b * D + dch);
                            } else if (!first) {
                                x = loadv<CV>(sbnd + q * kDc + cofs);
                            }
                        } else if (!first) {
                            x = loadv<CV>(ss + (q * Lc + ra - 1) * kDc + cofs);
                        }
                        if (!first) {
                            xa = loadv<CV>(ss + (q * Lc + ra) * kDc + cofs);
                            xb = loadv<CV>(ss + (q * Lc + rb) * kDc + cofs);
                        }
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) {
                            sp[q][jp] = make_float2(x.v[2 * jp], x.v[2 * jp + 1]);
                            ska[q][jp] = make_float2(xa.v[2 * jp], xa.v[2 * jp + 1]);
                            skb[q][jp] = make_float2(xb.v[2 * jp], xb.v[2 * jp + 1]);
                        }
                    }
                    float2 ua[G][NP], ub[G][NP];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        FV<CV> x = loadv<CV>(su + (ra * G + g) * kDc + cofs);
                        FV<CV> z = loadv<CV>(su + (rb * G + g) * kDc + cofs);
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) {
                            ua[g][jp] = make_float2(x.v[2 * jp], x.v[2 * jp + 1]);
                            ub[g][jp] = make_float2(z.v[2 * jp], z.v[2 * jp + 1]);
                        }
                    }
                    const bool va = (l0 + ra) < L && chv, vb = (l0 + rb) < L && chv;
                    Map2 agg2[NP];
                    float2 offa[NS][NP], offb[NS][NP];
#pragma unroll
                    for (int jp = 0; jp < NP; ++jp) {
                        float2 s_a[NS], s_b[NS], u_a[G], u_b[G], aa[G], fa[NS], fb[NS], ja[NS], jb[NS];
#pragma unroll
                        for (int q = 0; q < NS; ++q) {
                            s_a[q] = sp[q][jp];
                            s_b[q] = ska[q][jp];
                        }
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            u_a[g] = ua[g][jp];
                            u_b[g] = ub[g][jp];
                            aa[g] = wv[g][jp];
                        }
                        Map2 ea, eb;
                        Rows2::eval(s_a, u_a, s_b, u_b, aa, fa, fb, ea, eb);
                        if (first) {
#pragma unroll
                            for (int q = 0; q < NS; ++q) {
                                const float2 da = add2(ska[q][jp], neg2(fa[q]));
                                const float2 db = add2(skb[q][jp], neg2(fb[q]));
                                if (va) rpre = max_keep_nan(rpre, max_keep_nan(fabsf(da.x), fabsf(da.y)));
                                if (vb) rpre = max_keep_nan(rpre, max_keep_nan(fabsf(db.x), fabsf(db.y)));
                            }
                        }
                        apply_matrix2(ea, s_a, ja);
                        apply_matrix2(eb, s_b, jb);
                        float2 oa[NS], ob[NS];
#pragma unroll
                        for (int q = 0; q < NS; ++q) {
                            oa[q] = fma2(ja[q], bc2(-1.0f), fa[q]);
                            ob[q] = fma2(jb[q], bc2(-1.0f), fb[q]);
                            offa[q][jp] = oa[q];
                            offb[q][jp] = ob[q];
                        }
                        set_offset2(ea, oa);
                        set_offset2(eb, ob);
                        Jn[0][jp] = jacobian_of(ea);
                        Jn[1][jp] = jacobian_of(eb);
                        agg2[jp] = compose(eb, ea);
                    }
#pragma unroll
                    for (int q = 0; q < NS; ++q) {
                        float va4[CV], vb4[CV];
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) {
                            va4[2 * jp] = offa[q][jp].x;
                            va4[2 * jp + 1] = offa[q][jp].y;
                            vb4[2 * jp] = offb[q][jp].x;
                            vb4[2 * jp + 1] = offb[q][jp].y;
                        }
                        storev<CV>(ss + (q * Lc + ra) * kDc + cofs, va4);   // step a's state is no longer read
                        storev<CV>(slast + (q * CW + rp) * kDc + cofs, vb4);  // step b's state is the next pair's input
                    }
                    {
#pragma unroll
                        for (int i = 0; i < NC; ++i) {
                            float v4[CV];
#pragma unroll
                            for (int jp = 0; jp < NP; ++jp) {
                                v4[2 * jp] = agg2[jp].lane(0).get(i);
                                v4[2 * jp + 1] = agg2[jp].lane(1).get(i);
                            }
                            storev<CV>(sagg + (i * CW + rp) * kDc + cofs, v4);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar_aggr[wb]);
                }
                if (prev.x < p.n_tiles) {
                    // ---- sweep 2 of tile n-1
                    const int sp_ = (n - 1) % kStages, wp = (n - 1) % kWork;
                    (void)mbar_wait_bounded(&bar_carry[wp], uint32_t((n - 1) / kWork) & 1u, err, p.wait_ns);
                    const unsigned char* st = stage_at(sp_);
                    const unsigned char* wk = work_at(wp);
                    const UT* su = reinterpret_cast<const UT*>(st + LY::off_u);
                    const float* ss = reinterpret_cast<const float*>(st + LY::off_s);
                    const float* sa = reinterpret_cast<const float*>(st + LY::off_a);
                    const float* slast = reinterpret_cast<const float*>(wk + LY::off_last);
                    const float* spre = reinterpret_cast<const float*>(wk + LY::off_agg);
                    const float* car = reinterpret_cast<const float*>(wk + LY::off_carry);
                    const int c = prev.y, b = prev.z, d0 = prev.w;
                    const int l0 = c * Lc;
                    const int dch = d0 + cofs;
                    const bool chv = dch < D && !s_int[0];
                    float2 wv[G][NP];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        FV<CV> x = loadv<CV>(sa + g * kDc + cofs);
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) wv[g][jp] = make_float2(x.v[2 * jp], x.v[2 * jp + 1]);
                    }
                    // state entering this warp's steps = its prefix map applied to the tile's carry
                    float2 y0[NS][NP];
                    {
                        Map2 pre[NP];
#pragma unroll
                        for (int i = 0; i < NC; ++i) {
                            FV<CV> v = loadv<CV>(spre + (i * CW + rp) * kDc + cofs);
#pragma unroll
                            for (int jp = 0; jp < NP; ++jp) pre[jp].set(i, make_float2(v.v[2 * jp], v.v[2 * jp + 1]));
                        }
                        float2 ct[NS][NP];
#pragma unroll
                        for (int q = 0; q < NS; ++q) {
                            FV<CV> x = loadv<CV>(car + q * kDc + cofs);
#pragma unroll
                            for (int jp = 0; jp < NP; ++jp) ct[q][jp] = make_float2(x.v[2 * jp], x.v[2 * jp + 1]);
                        }
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) {
                            float2 x[NS], z[NS];
#pragma unroll
                            for (int q = 0; q < NS; ++q) x[q] = ct[q][jp];
                            apply2(pre[jp], x, z);
#pragma unroll
                            for (int q = 0; q < NS; ++q) y0[q][jp] = z[q];
                        }
                    }
                    // (PartialResiduals) Once a tile of this pass has found a residual
                    // above tol, the pass cannot end the solve with its
                    // residual reported (only a pass whose residual is <= tol,
                    // or the last allowed one, does), so the rest of its tiles
                    // leave the residual out -- unless a state it reads is not
                    // finite, which decides the outcome, and then the tile
                    // evaluates it.  Every decision stays the same; only the
                    // maxima of passes that continue are partial.
                    const bool skip_ok = PartialResiduals<Cell>::value && k + 1 < p.max_iters &&
                                         __shfl_sync(0xffffffffu, over_seen, 0) != 0;
                    float2 offa[NS][NP], offb[NS][NP], ua[G][NP], ub[G][NP];
#pragma unroll
                    for (int q = 0; q < NS; ++q) {
                        FV<CV> xa = loadv<CV>(ss + (q * Lc + ra) * kDc + cofs);
                        FV<CV> xb = loadv<CV>(slast + (q * CW + rp) * kDc + cofs);
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) {
                            offa[q][jp] = make_float2(xa.v[2 * jp], xa.v[2 * jp + 1]);
                            offb[q][jp] = make_float2(xb.v[2 * jp], xb.v[2 * jp + 1]);
                        }
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        FV<CV> x = loadv<CV>(su + (ra * G + g) * kDc + cofs);
                        FV<CV> z = loadv<CV>(su + (rb * G + g) * kDc + cofs);
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) {
                            ua[g][jp] = make_float2(x.v[2 * jp], x.v[2 * jp + 1]);
                            ub[g][jp] = make_float2(z.v[2 * jp], z.v[2 * jp + 1]);
                        }
                    }
                    const long long la = l0 + ra, lb = l0 + rb;
                    const bool va = la < L && chv, vb = lb < L && chv;
                    float2 ya[NS][NP], yb[NS][NP];
                    if constexpr (PartialResiduals<Cell>::value) {
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) {
                            float2 s0v[NS], sav[NS], t0[NS], t1[NS];
#pragma unroll
                            for (int q = 0; q < NS; ++q) s0v[q] = y0[q][jp];
                            apply_matrix2(Jp[0][jp], s0v, t0);
#pragma unroll
                            for (int q = 0; q < NS; ++q) sav[q] = add2(t0[q], offa[q][jp]);
                            apply_matrix2(Jp[1][jp], sav, t1);
#pragma unroll
                            for (int q = 0; q < NS; ++q) {
                                ya[q][jp] = sav[q];
                                yb[q][jp] = add2(t1[q], offb[q][jp]);
                            }
                        }
                        bool eval = !skip_ok;
                        if (skip_ok) {
                            bool finite = true;
#pragma unroll
                            for (int jp = 0; jp < NP; ++jp)
#pragma unroll
                                for (int q = 0; q < NS; ++q) {
                                    // (the state entering the warp's steps too:
                                    // a residual reads the state before its step)
                                    if (va) finite = finite && finite2(y0[q][jp]) && finite2(ya[q][jp]);
                                    if (vb) finite = finite && finite2(yb[q][jp]);
                                }
                            eval = !__all_sync(0xffffffffu, finite);
                        }
                        if (eval) {
                            float tmax = 0.f;
#pragma unroll
                            for (int jp = 0; jp < NP; ++jp) {
                                float2 s0v[NS], sav[NS], sbv[NS], u_a[G], u_b[G], aa[G], fa[NS], fb[NS];
#pragma unroll
                                for (int q = 0; q < NS; ++q) {
                                    s0v[q] = y0[q][jp];
                                    sav[q] = ya[q][jp];
                                    sbv[q] = yb[q][jp];
                                }
#pragma unroll
                                for (int g = 0; g < G; ++g) {
                                    u_a[g] = ua[g][jp];
                                    u_b[g] = ub[g][jp];
                                    aa[g] = wv[g][jp];
                                }
                                Rows2::value(s0v, u_a, sav, u_b, aa, fa, fb);
#pragma unroll
                                for (int q = 0; q < NS; ++q) {
                                    const float2 da = add2(sav[q], neg2(fa[q]));
                                    const float2 db = add2(sbv[q], neg2(fb[q]));
                                    if (va) tmax = max_keep_nan(tmax, max_keep_nan(fabsf(da.x), fabsf(da.y)));
                                    if (vb) tmax = max_keep_nan(tmax, max_keep_nan(fabsf(db.x), fabsf(db.y)));
                                }
                            }
                            rpost = max_keep_nan(rpost, tmax);
                            const bool above = !(tmax <= p.tol);  // NaN counts
                            if (p.skip_res && __any_sync(0xffffffffu, above) && !skip_ok && lane == 0)
                                atomicMax(&hdr->over[slot], 1u);
                        }
                    } else {
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) {
                            float2 s0v[NS], sav[NS], sbv[NS], u_a[G], u_b[G], aa[G], fa[NS], fb[NS], t0[NS], t1[NS];
#pragma unroll
                            for (int q = 0; q < NS; ++q) s0v[q] = y0[q][jp];
                            apply_matrix2(Jp[0][jp], s0v, t0);
#pragma unroll
                            for (int q = 0; q < NS; ++q) sav[q] = add2(t0[q], offa[q][jp]);
                            apply_matrix2(Jp[1][jp], sav, t1);
#pragma unroll
                            for (int q = 0; q < NS; ++q) sbv[q] = add2(t1[q], offb[q][jp]);
#pragma unroll
                            for (int g = 0; g < G; ++g) {
                                u_a[g] = ua[g][jp];
                                u_b[g] = ub[g][jp];
                                aa[g] = wv[g][jp];
                            }
                            Rows2::value(s0v, u_a, sav, u_b, aa, fa, fb);
#pragma unroll
                            for (int q = 0; q < NS; ++q) {
                                const float2 da = add2(sav[q], neg2(fa[q]));
                                const float2 db = add2(sbv[q], neg2(fb[q]));
                                if (va) rpost = max_keep_nan(rpost, max_keep_nan(fabsf(da.x), fabsf(da.y)));
                                if (vb) rpost = max_keep_nan(rpost, max_keep_nan(fabsf(db.x), fabsf(db.y)));
                                ya[q][jp] = sav[q];
                                yb[q][jp] = sbv[q];
                            }
                        }
                    }
#pragma unroll
                    for (int q = 0; q < NS; ++q) {
                        float oa4[CV], ob4[CV];
#pragma unroll
                        for (int jp = 0; jp < NP; ++jp) {
                            oa4[2 * jp] = ya[q][jp].x;
                            oa4[2 * jp + 1] = ya[q][jp].y;
                            ob4[2 * jp] = yb[q][jp].x;
                            ob4[2 * jp + 1] = yb[q][jp].y;
                        }
                        if (va) stcgv<CV>(p.st[q] + ((b * L + la) * D + dch), oa4);
                        if (vb) stcgv<CV>(p.st[q] + ((b * L + lb) * D + dch), ob4);
                        if (rp == CW - 1 && c + 1 < p.n_chunks && chv)
                            stcgv<CV>(p.bnd + ((((size_t)((k + 1) & 1) * NS + q) * p.B + b) * p.n_chunks + c) * Dpad +
                                          dch,
                                      ob4);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar_empty[sp_]);
                }
                if (!valid) break;
                prev = job;
#pragma unroll
                for (int r = 0; r < 2; ++r)
#pragma unroll
                    for (int jp = 0; jp < NP; ++jp) Jp[r][jp] = Jn[r][jp];
            }
        }

        // residual maxima of this CTA for this pass (max with NaN kept)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            rpost = max_keep_nan(rpost, __shfl_xor_sync(0xffffffffu, rpost, off));
            rpre = max_keep_nan(rpre, __shfl_xor_sync(0xffffffffu, rpre, off));
        }
        if (lane == 0) {
            s_red[w] = rpost;
            s_red[CWT + 1 + w] = rpre;
        }
        __syncthreads();
        if (tid == 0) {
            float a = 0.f, b2 = 0.f;
            for (int i = 0; i <= CWT; ++i) {
                a = max_keep_nan(a, s_red[i]);
                b2 = max_keep_nan(b2, s_red[CWT + 1 + i]);
            }
            // non-negative floats (and NaN) order like their bit patterns
            atomicMax(&hdr->res[slot], __float_as_uint(a) & 0x7fffffffu);
            if (first) atomicMax(&hdr->res0, __float_as_uint(b2) & 0x7fffffffu);
        }

        const bool bar_ok = grid_barrier(&hdr->bar, unsigned(k - k0), err, p.wait_ns, &s_int[1]);
        if (tid == 0) {
            // every CTA has finished pass k
            if (blockIdx.x == 0 && k + 1 < kPassTimes) hdr->t_pass[k + 1] = global_timer_ns();
            NewtonDecision d = newton_decide(hdr, k, slot, bar_ok, p.tol, p.max_iters);
            if (!d.cont && blockIdx.x == 0) newton_publish(hdr, d, k);
            s_int[2] = d.cont;
            s_int[3] = d.zero;
        }
        __syncthreads();
        if (!s_int[2]) {
            if (s_int[3]) newton_zero_states<NS>(p, tid, blockDim.x);
            return;
        }
        if (tid == 0) fence_proxy_async_global();  // other CTAs' state writes before our next TMA reads
    }
}

}  // namespace pararnn
