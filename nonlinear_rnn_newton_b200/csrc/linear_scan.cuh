// Plain diagonal linear scan: one pass of the chunked parallel scan over the
// linear recurrence of the zero-weight GRU,
//   h_l = (1 - s(u_z,l)) h_{l-1} + s(u_z,l) tanh(u_c,l),
// reading two of the three gate streams.  It is the linear SSM of the page
// "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala pra
// 7B parâmetros" (section "O compromisso que SSMs fizeram") and serves as the
// lower bound of one scan pass for the same [B][L][3][D] input: a Newton
// iteration cannot move fewer bytes than this.
//
// The kernel has the warp-specialised shape of the fused solve
// (newton_ws.cuh), without the Newton loop and the residual:
//   * CW compute warps, each owning R consecutive steps of a tile (tile =
//     R*CW steps x 128 channels).  For tile n a warp forms the step maps of
//     its R steps from the gates in the ring (kept in registers), folds them
//     and hands the fold to the control warp -- the ring stage is then free
//     -- and runs sweep 2 of tile n-1: its prefix applied to the tile's carry,
//     then the R states, stored straight to global memory.
//   * one control warp takes group tickets (two chunks of one sequence each),
//     issues the TMA loads of gates z and c into a ring, composes the folds
//     into exclusive prefixes in place, resolves the group's carry by the
//     look-back (stepping back over predecessors' aggregates, or waiting for
//     the predecessor's inclusive value), writes each tile's carry and then
//     refills the stage the tile came from.
// Every wait is bounded.
#pragma once

#include <climits>

#include "newton_ws.cuh"

namespace pararnn {

#ifndef PARARNN_LIN_STAGES
#define PARARNN_LIN_STAGES 4
#endif
constexpr int kLinStages = PARARNN_LIN_STAGES;  // TMA ring of the linear scan

struct LinScanParams {
    const float* h0;  // [B][D] or NULL
    float* h;         // [B][L][D]
    long long B, L, D;
    int S, n_chunks, n_tiles;
    int lb_walk;      // look-backs step back over aggregates (1) or wait for inclusive values (0)
    WsHeader* hdr;
    unsigned long long* desc;  // one descriptor per group of chunks (tagged words)
    unsigned long long wait_ns;
};

// CW compute warps of R steps each.
template <class UT, int CW, int R>
struct LinScanLayout {
    static constexpr int Lc = R * CW;
    static constexpr size_t a128(size_t x) { return (x + 127) & ~size_t(127); }
    static constexpr size_t g_tx = size_t(Lc) * kDc * sizeof(UT);  // one gate stream of a tile
    static constexpr size_t off_c = a128(g_tx);                    // ring stage: gate z | gate c
    static constexpr size_t stage_bytes = 2 * a128(g_tx);
    // work buffer: folds, then exclusive prefixes [2][CW][kDc] | tile carry [kDc]
    static constexpr size_t off_agg = 0;
    static constexpr size_t off_carry = a128(size_t(2) * CW * kDc * 4);
    static constexpr size_t work_bytes = off_carry + a128(size_t(kDc) * 4);
    static constexpr size_t off_work = kLinStages * stage_bytes;
    static constexpr size_t off_misc = off_work + kWork * work_bytes;
    // misc: a job (ticket, chunk, batch row, first channel) per stage (16-byte
    // aligned), barriers (full per stage; aggr, carry per work buffer), 4 flags
    static constexpr size_t misc_bytes = a128(kLinStages * 16 + (kLinStages + 2 * kWork) * 8 + 4 * 4);
    static constexpr size_t smem_bytes = off_misc + misc_bytes;
    static constexpr int threads = 32 * (CW + 1);
    static constexpr int desc_words = TileDesc<Aff<1>, 1>::words;
    static_assert(smem_bytes <= 232448, "shared memory");
    static_assert(R >= 2 && R % 2 == 0 && CW >= 1, "tile: steps of a warp come in pairs");
    static_assert(kLinStages >= 2, "ring");
};

// The step maps of the zero-weight GRU, (1 - z, z tanh(c)), of two steps a
// and b on a channel pair; the two steps share one reciprocal per channel.
__device__ __forceinline__ void linear_gru_maps2(float2 uza, float2 uca, float2 uzb, float2 ucb, Aff2<1>& ma,
                                                 Aff2<1>& mb)
{
    float2 za, ta, zb, tb;
    sigmoid_tanh4_2(uza, uca, uzb, ucb, za, ta, zb, tb);
    ma = {add2(bc2(1.0f), neg2(za)), mul2(za, ta)};
    mb = {add2(bc2(1.0f), neg2(zb)), mul2(zb, tb)};
}

// LB: look-backs step back over aggregates (1), wait for inclusive values (0)
// or follow p.lb_walk (2).
template <class UT, int CW, int R, int LB = 2>
__global__ void __launch_bounds__(32 * (CW + 1), 1)
    linear_scan_kernel(const __grid_constant__ CUtensorMap tm_u, const LinScanParams p)
{
    using LY = LinScanLayout<UT, CW, R>;
    using Map = Aff<1>;
    using Map2 = Aff2<1>;
    constexpr int Lc = LY::Lc, NP = kV / 2;
    const bool walk = LB == 2 ? p.lb_walk != 0 : LB == 1;

    extern __shared__ __align__(128) unsigned char smem[];
    int4* s_job = reinterpret_cast<int4*>(smem + LY::off_misc);         // [kLinStages]
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(s_job + kLinStages);  // [kLinStages]
    uint64_t* bar_aggr = bar_full + kLinStages;                          // [kWork]
    uint64_t* bar_carry = bar_aggr + kWork;                              // [kWork]
    int* s_int = reinterpret_cast<int*>(bar_carry + kWork);              // flags
    auto stage_at = [&](int i) { return smem + i * LY::stage_bytes; };
    auto work_at = [&](int i) { return smem + LY::off_work + i * LY::work_bytes; };

    const int tid = threadIdx.x;
    const int w = tid >> 5;
    const int lane = tid & 31;
    WsHeader* hdr = p.hdr;
    int* err = &hdr->error;
    const long long D = p.D, L = p.L;
    const int BS = int(p.B) * p.S;

    if (tid == 0) {
        prefetch_tensormap(&tm_u);
        for (int i = 0; i < kLinStages; ++i) mbar_init(&bar_full[i], 1);
        for (int i = 0; i < kWork; ++i) {
            mbar_init(&bar_aggr[i], CW);
            mbar_init(&bar_carry[i], 1);
        }
        s_int[0] = 0;  // look-back failure seen by the control warp
        fence_mbar_init();
    }
    __syncthreads();

    if (w == CW) {
        // ---------------------------------------------------- control warp
        // (lane 0 only.)  A stage is refilled once every compute warp has
        // arrived on the tile's aggr barrier, after its last read of the
        // stage.  A look-back that gave up stops the loads; another CTA's
        // error reaches this one through its own bounded waits.
        auto issue = [&](int4 job, int stage) {
            if (s_int[0]) job.x = INT_MAX;
            if (job.x < p.n_tiles) {
                s_job[stage] = job;
                unsigned char* st = stage_at(stage);
                const int c = job.y, b = job.z, d0 = job.w;
                mbar_arrive_expect_tx(&bar_full[stage], uint32_t(2 * LY::g_tx));
                tma_load_4d(st, &tm_u, d0, 0, c * Lc, b, &bar_full[stage]);               // gate z
                tma_load_4d(st + LY::off_c, &tm_u, d0, 2, c * Lc, b, &bar_full[stage]);  // gate c
            } else {
                s_job[stage] = make_int4(INT_MAX, 0, 0, 0);
                mbar_arrive(&bar_full[stage]);
            }
        };
        // the next tile (ticket, chunk, batch row, first channel): the rest
        // of the current group, then a new group (a group ticket is taken only
        // when its first tile is issued); the divisions are taken once per
        // group (lane 0 only).
        const int n_groups = ((p.n_chunks + kGroup - 1) / kGroup) * BS;
        int g_c = 0, g_end = 0, g_q = 0, g_b = 0, g_d0 = 0;
        auto next_tile = [&]() {
            if (g_c >= g_end) {
                const int gt = int(atomicAdd(&hdr->tick[0], 1u));
                if (gt >= n_groups) return make_int4(INT_MAX, 0, 0, 0);
                const int gc = gt / BS;
                g_q = gt - gc * BS;
                g_c = gc * kGroup;
                g_end = min(g_c + kGroup, p.n_chunks);
                g_b = g_q / p.S;
                g_d0 = (g_q - g_b * p.S) * kDc;
            }
            const int c = g_c++;
            return make_int4(c * BS + g_q, c, g_b, g_d0);
        };
        if (lane == 0) {
#pragma unroll 1
            for (int i = 0; i < kLinStages; ++i) issue(next_tile(), i);
        }
        __syncwarp();
        // (the jobs in s_job are written by lane 0 and read by the warp after
        // a __syncwarp; a stage's job stays until the stage is refilled)
        auto refill = [&](int s) {
            if (lane == 0) issue(next_tile(), s);
            __syncwarp();
        };
        // folds of work buffer `wkb` -> exclusive prefixes (in place); the
        // tile's aggregate (the last inclusive prefix) in `run`.  The folds
        // are read in batches of five, so that the reads are in flight
        // together and only the compositions form a chain.
        auto prefix = [&](int wkb, Map (&run)[kV]) {
            float* agg = reinterpret_cast<float*>(work_at(wkb) + LY::off_agg) + lane * kV;
            constexpr int BT = 5;
#pragma unroll
            for (int j = 0; j < kV; ++j) run[j] = Map::identity();
#pragma unroll
            for (int s0 = 0; s0 < CW; s0 += BT) {
                F4 m[BT], v[BT];
#pragma unroll
                for (int i = 0; i < BT; ++i) {
                    if (s0 + i < CW) {
                        m[i] = load4(agg + (s0 + i) * kDc);
                        v[i] = load4(agg + (CW + s0 + i) * kDc);
                    }
                }
#pragma unroll
                for (int i = 0; i < BT; ++i) {
                    if (s0 + i < CW) {
                        float pm[kV], pv[kV];
#pragma unroll
                        for (int j = 0; j < kV; ++j) {
                            pm[j] = run[j].m;
                            pv[j] = run[j].v;
                            run[j] = compose(Map{m[i].v[j], v[i].v[j]}, run[j]);
                        }
                        store4(agg + (s0 + i) * kDc, pm);
                        store4(agg + (CW + s0 + i) * kDc, pv);
                    }
                }
            }
        };
        float y_inc[kV];  // state leaving the last tile handled here
        bool pre_done = false;  // the group's second tile's prefixes are computed (run_pre)
        Map run_pre[kV];
        for (int n = 0;; ++n) {
            const int s = n % kLinStages, wb = n % kWork;
            const int4 job = s_job[s];
            const int ticket = job.x;
            if (ticket >= p.n_tiles) break;
            const int c = job.y, b = job.z, d0 = job.w;
            const int rem = ticket - c * BS;  // sequence (batch row, slab)
            const int dch = d0 + lane * kV;
            const bool local = (c % kGroup) != 0;    // the group's second tile
            const int gt = (c / kGroup) * BS + rem;  // group ticket (descriptor index)
            LookbackProbe<Map, 1> pr;
            bool ok = true;
            Map run[kV];
            if (local && pre_done) {
#pragma unroll
                for (int j = 0; j < kV; ++j) run[j] = run_pre[j];
            } else {
                ok = mbar_wait_bounded(&bar_aggr[wb], uint32_t(n / kWork) & 1u, err, p.wait_ns);
                // first look-back read (issued only now, so that it sees
                // predecessors as late as possible)
                if (c > 0 && !local) {
                    if (walk) lookback_probe<Map, 1, true>(pr, gt - BS, p.desc, lane);
                    else lookback_probe<Map, 1, false>(pr, gt - BS, p.desc, lane);
                }
                prefix(wb, run);
            }
            float y[kV];
            if (local) {
#pragma unroll
                for (int j = 0; j < kV; ++j) y[j] = y_inc[j];
                pre_done = false;
            } else {
                // the group's second tile (next in the ring): its prefixes
                // now, while the look-back read is in flight
                bool two = false;
                if (c + 1 < p.n_chunks) {
                    const int n1 = n + 1;
                    if (s_job[n1 % kLinStages].x == ticket + BS) {
                        ok = mbar_wait_bounded(&bar_aggr[n1 % kWork], uint32_t(n1 / kWork) & 1u, err, p.wait_ns) &&
                             ok;
                        prefix(n1 % kWork, run_pre);
                        pre_done = two = true;
                    } else {
                        ok = false;  // a group's tiles are always issued back to back
                    }
                }
                float yq[1][kV];
                if (c > 0) {
                    if (walk) {
                        // the group's aggregate (both tiles' maps composed)
                        // goes out first, for look-backs that step over it
                        Map gagg[kV];
#pragma unroll
                        for (int j = 0; j < kV; ++j) gagg[j] = two ? compose(run_pre[j], run[j]) : run[j];
                        publish_aggregate<Map, 1>(p.desc, gt, 0, gagg, lane);
                        ok = lookback_resolve<Map, 1, true>(gt, BS, 0, yq, p.desc, lane, err, p.wait_ns, pr) && ok;
                    } else {
                        ok = lookback_resolve<Map, 1, false>(gt, BS, 0, yq, p.desc, lane, err, p.wait_ns, pr) && ok;
                    }
                } else {
                    F4 x{{0.f, 0.f, 0.f, 0.f}};
                    if (dch < D && p.h0) x = load4(p.h0 + b * D + dch);
#pragma unroll
                    for (int j = 0; j < kV; ++j) yq[0][j] = x.v[j];
                }
#pragma unroll
                for (int j = 0; j < kV; ++j) y[j] = yq[0][j];
            }
            // the state leaving this tile; at a group's head, also the state
            // leaving the group (its inclusive value)
#pragma unroll
            for (int j = 0; j < kV; ++j) apply(run[j], &y[j], &y_inc[j]);
            const bool all_ok = __all_sync(0xffffffffu, ok);
            if (!local && all_ok) {
                float incl[1][kV];
#pragma unroll
                for (int j = 0; j < kV; ++j) {
                    incl[0][j] = y_inc[j];
                    if (pre_done) apply(run_pre[j], &y_inc[j], &incl[0][j]);
                }
                publish_inclusive<Map, 1>(p.desc, gt, 0, incl, lane);
            }
            store4(reinterpret_cast<float*>(work_at(wb) + LY::off_carry) + lane * kV, y);
            if (!all_ok && lane == 0) s_int[0] = 1;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_carry[wb]);
            // every compute warp was done with tile n's stage when it arrived
            // on the tile's aggr barrier: the stage takes the next load
            refill(s);
        }
    } else {
        // ---------------------------------------------------- compute warps
        const int cofs = lane * kV;  // first channel of this lane in the tile
        const int r0 = w * R;        // this warp's first step in the tile
        int4 prev = make_int4(INT_MAX, 0, 0, 0);  // job of the previous tile
        // one tile: sweep 1 of tile n into `cur`, then sweep 2 of tile n-1
        // from `prv`; false once the ring runs dry
        auto tile = [&](int n, Map2 (&cur)[R][NP], const Map2 (&prv)[R][NP]) -> bool {
            const int s = n % kLinStages, wb = n % kWork;
            (void)mbar_wait_bounded(&bar_full[s], uint32_t(n / kLinStages) & 1u, err, p.wait_ns);
            const int4 job = s_job[s];
            const bool valid = job.x < p.n_tiles;
            if (valid) {
                const UT* sz = reinterpret_cast<const UT*>(stage_at(s));
                const UT* sc = reinterpret_cast<const UT*>(stage_at(s) + LY::off_c);
                Map2 agg[NP];
#pragma unroll
                for (int jp = 0; jp < NP; ++jp) agg[jp] = Map2::identity();
#pragma unroll
                for (int r = 0; r < R; r += 2) {
                    const FV<kV> za = loadv<kV>(sz + (r0 + r) * kDc + cofs);
                    const FV<kV> ga = loadv<kV>(sc + (r0 + r) * kDc + cofs);
                    const FV<kV> zb = loadv<kV>(sz + (r0 + r + 1) * kDc + cofs);
                    const FV<kV> gb = loadv<kV>(sc + (r0 + r + 1) * kDc + cofs);
#pragma unroll
                    for (int jp = 0; jp < NP; ++jp) {
                        linear_gru_maps2(make_float2(za.v[2 * jp], za.v[2 * jp + 1]),
                                         make_float2(ga.v[2 * jp], ga.v[2 * jp + 1]),
                                         make_float2(zb.v[2 * jp], zb.v[2 * jp + 1]),
                                         make_float2(gb.v[2 * jp], gb.v[2 * jp + 1]), cur[r][jp], cur[r + 1][jp]);
                        agg[jp] = compose(cur[r + 1][jp], compose(cur[r][jp], agg[jp]));
                    }
                }
                float* sagg = reinterpret_cast<float*>(work_at(wb) + LY::off_agg);
                float m4[kV], v4[kV];
#pragma unroll
                for (int jp = 0; jp < NP; ++jp) {
                    m4[2 * jp] = agg[jp].m.x;
                    m4[2 * jp + 1] = agg[jp].m.y;
                    v4[2 * jp] = agg[jp].v.x;
                    v4[2 * jp + 1] = agg[jp].v.y;
                }
                storev<kV>(sagg + w * kDc + cofs, m4);
                storev<kV>(sagg + (CW + w) * kDc + cofs, v4);
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_aggr[wb]);  // also releases the stage
            }
            if (prev.x < p.n_tiles) {
                const int wp = (n - 1) % kWork;
                (void)mbar_wait_bounded(&bar_carry[wp], uint32_t((n - 1) / kWork) & 1u, err, p.wait_ns);
                const float* spre = reinterpret_cast<const float*>(work_at(wp) + LY::off_agg);
                const float* car = reinterpret_cast<const float*>(work_at(wp) + LY::off_carry);
                const int c = prev.y, b = prev.z, d0 = prev.w;
                const long long l0 = (long long)c * Lc + r0;
                const int dch = d0 + cofs;
                const bool chv = dch < D && !s_int[0];
                const FV<kV> pm = loadv<kV>(spre + w * kDc + cofs);
                const FV<kV> pv = loadv<kV>(spre + (CW + w) * kDc + cofs);
                const FV<kV> cr = loadv<kV>(car + cofs);
                float2 y[NP];
#pragma unroll
                for (int jp = 0; jp < NP; ++jp)
                    y[jp] = fma2(make_float2(pm.v[2 * jp], pm.v[2 * jp + 1]), make_float2(cr.v[2 * jp], cr.v[2 * jp + 1]),
                                 make_float2(pv.v[2 * jp], pv.v[2 * jp + 1]));
                float* dst = p.h + ((b * L + l0) * D + dch);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    float o4[kV];
#pragma unroll
                    for (int jp = 0; jp < NP; ++jp) {
                        y[jp] = fma2(prv[r][jp].m, y[jp], prv[r][jp].v);
                        o4[2 * jp] = y[jp].x;
                        o4[2 * jp + 1] = y[jp].y;
                    }
                    if (chv && l0 + r < L) stcgv<kV>(dst + r * D, o4);
                }
            }
            prev = job;
            return valid;
        };
        // two map sets alternate between the tiles, so nothing is copied
        Map2 ma[R][NP], mb[R][NP];
        for (int n = 0;; n += 2) {
            if (!tile(n, ma, mb)) break;
            if (!tile(n + 1, mb, ma)) break;
        }
    }
}

}  // namespace pararnn
