// Fused ParaRNN Newton solve: one cooperative kernel runs every Newton
// iteration of a ParaGRU (scalar Jacobian) or ParaLSTM (2x2 Jacobian) solve.
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros".
//   "A sacada: método de Newton": the unknowns are all states H; iteration k
//     evaluates F_l(H^k) = s_l - f(s_{l-1}, u_l) and J_l = df/ds_{l-1}, and
//     solves the linear SSM delta_l = J_l delta_{l-1} - F_l (delta_0 = 0) by
//     a parallel scan; H^{k+1} = H^k + delta.
//   "O compromisso que SSMs fizeram": the scan combines affine maps
//     associatively (tree order instead of step order).
//   "Engenharia pra escalar": diagonal / 2x2 Jacobians; Newton iterations,
//     system assembly and the parallel reduction fused in one kernel.
//
// Work decomposition.  A tile is (batch b, slab of kDc = 128 channels, chunk
// of Lc = 8*T timesteps).  Tiles are handed out in ticket order (chunk-major)
// from an atomic counter, so every tile's predecessor along the sequence has
// a smaller ticket and is already owned by a running CTA.  Per tile:
//   1. TMA loads the gate tile [Lc][G][128] and the state tile(s) [Lc][128]
//      into shared memory (one mbarrier).
//   2. Sweep 1: warp w owns rows w*T..w*T+T-1, lane owns 4 channels; each
//      thread evaluates the cell and its Jacobian per element, keeps J_l in
//      registers, writes the offset o_l = f_l - J_l s^k_{l-1} over the state
//      tile, and folds its T affine maps s -> J_l s + o_l into one (the
//      Newton step in direct form: s^{k+1}_l = J_l s^{k+1}_{l-1} + o_l equals
//      s^k_l + delta_l).
//   3. Each warp publishes its segment's map in shared memory; warp w
//      composes segments 0..w-1 into its exclusive prefix, warp 0 composes
//      all of them into the tile aggregate.
//   4. Decoupled look-back (warp 0): publish the aggregate, walk back over
//      predecessors' aggregates until an inclusive prefix is found, publish
//      the inclusive value.  Tagged 64-bit words, no fences, bounded waits.
//   5. Sweep 2: one FMA per element gives s^{k+1} from the incoming state;
//      write H^{k+1} in place and evaluate the residual of the *updated*
//      states (no extra memory traffic) for the convergence test.
// The value of the state just before a chunk is kept in a small ping-pong
// boundary array, so the in-place update never races with a neighbour.
// Tiles flow through a two-stage shared-memory ring: thread 0 starts the TMA
// loads of the tile after next as soon as every warp has released its stage
// (an mbarrier each warp arrives on), so copies overlap compute and only two
// CTA-wide barriers remain per tile.  Between iterations a grid barrier; every
// CTA reads the global residual and takes the same decision, so the loop
// needs no host round trip.
#pragma once

#include <climits>

#include "scan_common.cuh"

namespace pararnn {

struct NewtonParams {
    const float* a;         // [G][D]
    const float* s0[2];     // initial state per component [B][D] (NULL = zeros)
    float* st[2];           // states per component [B][L][D]
    long long B, L, D;
    int S;                  // channel slabs per batch row
    int n_chunks;           // chunks along L
    int n_tiles;            // n_chunks * B * S
    float tol;
    int max_iters;
    WsHeader* hdr;
    unsigned long long* desc;  // [n_tiles][desc_words] tagged words
    float* bnd;             // [2][NS][B][n_chunks][S*kDc]
    unsigned long long wait_ns;
};


// Convergence decision after pass k, taken identically by every CTA from the
// global residual maxima (see the stopping rule in pararnn.h).
struct NewtonDecision {
    int cont;    // run another pass
    int zero;    // return the initial guess H^0 = 0
    int iters, status;
    float residual, residual0;
};

__device__ __forceinline__ NewtonDecision newton_decide(WsHeader* hdr, int k, int slot, bool bar_ok, float tol,
                                                        int max_iters)
{
    NewtonDecision d{0, 0, k + 1, PARARNN_OK, 0.f, 0.f};
    const unsigned post_bits = ld_acquire_gpu_u32(&hdr->res[slot]);
    const unsigned pre_bits = ld_acquire_gpu_u32(&hdr->res0);
    const float r0 = __uint_as_float(pre_bits);
    const float rk = __uint_as_float(post_bits);
    const int e = ld_relaxed_gpu(&hdr->error);
    d.residual0 = r0;
    d.residual = rk;
    if (!bar_ok || e != 0) {
        d.status = e != 0 ? e : PARARNN_ERR_TIMEOUT;
        return d;
    }
    if (k == 0) {
        if (pre_bits >= 0x7f800000u) {  // NaN or inf residual of the initial guess
            d.status = PARARNN_ERR_NONFINITE;
            d.iters = 0;
            d.residual = r0;
            d.zero = 1;
            return d;
        }
        if (r0 <= tol || max_iters == 0) {
            d.status = r0 <= tol ? PARARNN_OK : PARARNN_NOT_CONVERGED;
            d.iters = 0;
            d.residual = r0;
            d.zero = 1;
            return d;
        }
    }
    if (post_bits >= 0x7f800000u) d.status = PARARNN_ERR_NONFINITE;
    else if (rk <= tol) d.status = PARARNN_OK;
    else if (k + 1 >= max_iters) d.status = PARARNN_NOT_CONVERGED;
    else d.cont = 1;
    return d;
}

__device__ __forceinline__ void newton_publish(WsHeader* hdr, const NewtonDecision& d, int k)
{
    hdr->result.status = d.status;
    hdr->result.iters = d.iters;
    hdr->result.residual = d.residual;
    hdr->result.residual0 = d.residual0;
    hdr->passes = k + 1;
}

// Converged (or stopped) at the initial guess: the states are H^0 = 0.
template <int NS>
__device__ __forceinline__ void newton_zero_states(const NewtonParams& p, int tid, int nthreads)
{
    const size_t n4 = size_t(p.B * p.L * p.D) / 4;
    for (int q = 0; q < NS; ++q) {
        float4* o = reinterpret_cast<float4*>(p.st[q]);
        for (size_t i = size_t(blockIdx.x) * nthreads + tid; i < n4; i += size_t(gridDim.x) * nthreads)
            o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

template <class Cell, class UT, int T>
struct NewtonLayout {
    static constexpr int G = Cell::G;
    static constexpr int NS = Cell::NS;
    static constexpr int NC = Cell::Map::kFloats;
    static constexpr int Lc = kWarps * T;
    static constexpr size_t u_bytes = size_t(Lc) * G * kDc * sizeof(UT);
    static constexpr size_t s_bytes = size_t(Lc) * kDc * sizeof(float);
    // offsets of each warp's last row (kept apart so that the next warp can
    // still read that row's state from the tile)
    static constexpr size_t last_bytes = size_t(NS) * kWarps * kDc * sizeof(float);
    // two pipeline stages, each [gates][states / offsets][last-row offsets]
    static constexpr size_t stage_bytes = u_bytes + NS * s_bytes + last_bytes;
    static constexpr size_t off_scan = 2 * stage_bytes;  // per-warp aggregates [NC][kWarps][kScanPad]
    static constexpr size_t off_carry = off_scan + size_t(NC) * kWarps * kScanPad * 4;  // [NS][kDc]
    static constexpr size_t off_misc = off_carry + size_t(NS) * kDc * 4;
    // misc: 2 barriers per stage (32 B), 16 flags (64 B), 2*kWarps residual slots
    static constexpr size_t smem_bytes = off_misc + ((96 + 8 * kWarps + 127) / 128) * 128;
    static constexpr int desc_words = TileDesc<typename Cell::Map, NS>::words;
    static_assert(smem_bytes <= 232448, "shared memory");
    static_assert(u_bytes % 128 == 0 && stage_bytes % 128 == 0 && off_scan % 16 == 0, "alignment");
};

template <class Cell, class UT, int T>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
    newton_solve_kernel(const __grid_constant__ CUtensorMap tm_u,
                        const __grid_constant__ CUtensorMap tm_s0,
                        const __grid_constant__ CUtensorMap tm_s1, const NewtonParams p)
{
    using LY = NewtonLayout<Cell, UT, T>;
    using Map = typename Cell::Map;
    using Packed = typename Cell::Packed;
    using Map2 = typename Packed::Map2;
    constexpr int G = LY::G, NS = LY::NS, NC = LY::NC, Lc = LY::Lc;

    extern __shared__ __align__(128) unsigned char smem[];
    float* scan = reinterpret_cast<float*>(smem + LY::off_scan);    // [NC][kWarps][kScanPad]
    float* scarry = reinterpret_cast<float*>(smem + LY::off_carry);  // [NS][kDc]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + LY::off_misc);         // per stage: loads landed
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + LY::off_misc + 16);   // per stage: all warps done
    int* s_int = reinterpret_cast<int*>(smem + LY::off_misc + 32);             // [0..1] tickets per stage
    unsigned* s_red = reinterpret_cast<unsigned*>(smem + LY::off_misc + 96);

    const int tid = threadIdx.x;
    const int w = tid >> 5;
    const int lane = tid & 31;
    WsHeader* hdr = p.hdr;
    int* err = &hdr->error;
    const long long D = p.D, L = p.L;
    const int BS = int(p.B) * p.S;
    const int Dpad = p.S * kDc;

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&empty[0], kWarps);
        mbar_init(&empty[1], kWarps);
        fence_mbar_init();
        prefetch_tensormap(&tm_u);
        prefetch_tensormap(&tm_s0);
        if (NS == 2) prefetch_tensormap(&tm_s1);
    }
    __syncthreads();
    uint32_t full_par = 0;   // all threads: bit s = parity of stage s's next "full" completion
    uint32_t empty_par = 0;  // thread 0: bit s = parity of stage s's next "empty" completion
    uint32_t used = 0;       // thread 0: bit s = stage s holds a tile not yet released

    // Thread 0: put tile t into `stage`: wait until every warp has released the
    // stage, record the ticket, start the TMA loads (or, past the last tile,
    // just complete the stage's phase so the consumers see the end).
    auto issue = [&](int t, int stage, bool first) {
        if (used & (1u << stage)) {
            (void)mbar_wait_bounded(&empty[stage], (empty_par >> stage) & 1u, err, p.wait_ns);
            empty_par ^= 1u << stage;
            used &= ~(1u << stage);
        }
        if (error_raised(err)) t = INT_MAX;
        s_int[stage] = t;
        if (t < p.n_tiles) {
            const int c = t / BS, rem = t - (t / BS) * BS;
            const int b = rem / p.S, d0 = (rem - b * p.S) * kDc;
            unsigned char* st = smem + stage * LY::stage_bytes;
            fence_proxy_async_shared();  // the warps' generic smem accesses before the async writes
            const uint32_t bytes = uint32_t(LY::u_bytes + (first ? 0 : NS * LY::s_bytes));
            mbar_arrive_expect_tx(&full[stage], bytes);
            tma_load_4d(st, &tm_u, d0, 0, c * Lc, b, &full[stage]);
            if (!first) {
                tma_load_3d(st + LY::u_bytes, &tm_s0, d0, c * Lc, b, &full[stage]);
                if (NS == 2) tma_load_3d(st + LY::u_bytes + LY::s_bytes, &tm_s1, d0, c * Lc, b, &full[stage]);
            }
            used |= 1u << stage;
        } else {
            mbar_arrive(&full[stage]);
        }
    };

    for (int k = 0;; ++k) {
        const int slot = k % 3;
        if (blockIdx.x == 0 && tid == 0) {
            // slot (k+1)%3 was last used two passes ago; every CTA is past it
            hdr->tick[(k + 1) % 3] = 0u;
            hdr->res[(k + 1) % 3] = 0u;
        }
        const bool first = (k == 0);
        unsigned rpost = 0u, rpre = 0u;

        // Tickets run one tile ahead of the loads, the loads one tile ahead of
        // the compute: the atomic's latency and the copies overlap the work.
        int tnext = 0;
        if (tid == 0) {
            issue(int(atomicAdd(&hdr->tick[slot], 1u)), 0, first);
            tnext = int(atomicAdd(&hdr->tick[slot], 1u));
        }
        int stage = 0;
        for (;;) {
            if (tid == 0) {
                issue(tnext, stage ^ 1, first);
                tnext = int(atomicAdd(&hdr->tick[slot], 1u));  // consumed at the next tile
            }
            (void)mbar_wait_bounded(&full[stage], (full_par >> stage) & 1u, err, p.wait_ns);
            full_par ^= 1u << stage;
            const int ticket = s_int[stage];
            if (ticket >= p.n_tiles) break;

            UT* su = reinterpret_cast<UT*>(smem + stage * LY::stage_bytes);
            float* ss = reinterpret_cast<float*>(smem + stage * LY::stage_bytes + LY::u_bytes);  // [NS][Lc][kDc]
            float* slast = ss + NS * Lc * kDc;                                                    // [NS][kWarps][kDc]

            const int c = ticket / BS;
            const int rem = ticket - c * BS;
            const int b = rem / p.S;
            const int sl = rem - b * p.S;
            const int l0 = c * Lc;
            const int d0 = sl * kDc;
            const int dch = d0 + lane * kV;
            const bool chv = dch < D;
            // this lane's 4 channels as two packed pairs (channels 0,1 and 2,3)
            float2 wv[G][2];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                F4 x = chv ? load4(p.a + g * D + dch) : F4{{0.f, 0.f, 0.f, 0.f}};
                wv[g][0] = make_float2(x.v[0], x.v[1]);
                wv[g][1] = make_float2(x.v[2], x.v[3]);
            }

            // 2. Sweep 1: evaluate cell, Jacobian and (pass 0) residual at H^k,
            //    keep J_l in registers, write the direct-form offset
            //    o_l = f_l - J_l s^k_{l-1}, and fold each thread's T maps
            //    (J_l, o_l): s^{k+1}_l = J_l s^{k+1}_{l-1} + o_l.  The offsets go
            //    over the state tile (s^k_l is dead once read), except the warp's
            //    last row, which the next warp still reads as its previous state.
            const int r0 = w * T;
            float2 sp[NS][2];  // s^k at the row before the current one
#pragma unroll
            for (int q = 0; q < NS; ++q) {
                F4 x{{0.f, 0.f, 0.f, 0.f}};
                if (w == 0) {
                    if (chv) {
                        if (c == 0) {
                            if (p.s0[q]) x = load4(p.s0[q] + b * D + dch);
                        } else if (!first) {
                            x = ldcg4(p.bnd + ((((size_t)(k & 1) * NS + q) * p.B + b) * p.n_chunks + (c - 1)) *
                                                  Dpad + dch);
                        }
                    }
                } else if (!first) {
                    x = load4(ss + (q * Lc + r0 - 1) * kDc + lane * kV);
                }
                sp[q][0] = make_float2(x.v[0], x.v[1]);
                sp[q][1] = make_float2(x.v[2], x.v[3]);
            }
            float init[NS][kV];  // state entering the tile if it is the sequence's first chunk
#pragma unroll
            for (int q = 0; q < NS; ++q) {
                init[q][0] = sp[q][0].x;
                init[q][1] = sp[q][0].y;
                init[q][2] = sp[q][1].x;
                init[q][3] = sp[q][1].y;
            }

            Map2 agg[2];
            typename Packed::Jac2 Jr[T][2];
            agg[0] = agg[1] = Map2::identity();
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const int row = r0 + t;
                float2 u[G][2];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    F4 x = load4(su + (row * G + g) * kDc + lane * kV);
                    u[g][0] = make_float2(x.v[0], x.v[1]);
                    u[g][1] = make_float2(x.v[2], x.v[3]);
                }
                float2 sk[NS][2], off[NS][2];
#pragma unroll
                for (int q = 0; q < NS; ++q) {
                    F4 x{{0.f, 0.f, 0.f, 0.f}};
                    if (!first) x = load4(ss + (q * Lc + row) * kDc + lane * kV);
                    sk[q][0] = make_float2(x.v[0], x.v[1]);
                    sk[q][1] = make_float2(x.v[2], x.v[3]);
                }
#pragma unroll
                for (int jp = 0; jp < 2; ++jp) {
                    float2 sv[NS], uu[G], aa[G], f[NS], js[NS];
#pragma unroll
                    for (int q = 0; q < NS; ++q) sv[q] = sp[q][jp];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        uu[g] = u[g][jp];
                        aa[g] = wv[g][jp];
                    }
                    Map2 e;
                    Packed::eval(sv, uu, aa, f, e);
                    if (first && (l0 + row) < L && chv) {
#pragma unroll
                        for (int q = 0; q < NS; ++q)
                            rpre = max(rpre, max(abs_bits(sk[q][jp].x - f[q].x), abs_bits(sk[q][jp].y - f[q].y)));
                    }
                    apply_matrix2(e, sv, js);
                    float2 o[NS];
#pragma unroll
                    for (int q = 0; q < NS; ++q) {
                        o[q] = fma2(js[q], bc2(-1.0f), f[q]);
                        off[q][jp] = o[q];
                        sp[q][jp] = sk[q][jp];
                    }
                    set_offset2(e, o);
                    Jr[t][jp] = jacobian_of(e);
                    agg[jp] = compose(e, agg[jp]);
                }
#pragma unroll
                for (int q = 0; q < NS; ++q) {
                    float v4[kV] = {off[q][0].x, off[q][0].y, off[q][1].x, off[q][1].y};
                    float* dst = (t == T - 1) ? slast + (q * kWarps + w) * kDc : ss + (q * Lc + row) * kDc;
                    store4(dst + lane * kV, v4);
                }
            }

            // 3. Combine the warps' segments: publish each warp's aggregate;
            //    warp w's exclusive prefix composes segments 0..w-1; warp 0 also
            //    composes the whole tile for the look-back.
            {
                Map a1[kV] = {agg[0].lane(0), agg[0].lane(1), agg[1].lane(0), agg[1].lane(1)};
                scan_put(scan, w, lane, a1);
            }
            __syncthreads();
            Map ex[kV];
#pragma unroll
            for (int j = 0; j < kV; ++j) ex[j] = Map::identity();
            const int nseg = (w == 0) ? kWarps : w;
            for (int seg = 0; seg < nseg; ++seg) {
                Map m[kV];
#pragma unroll
                for (int i = 0; i < NC; ++i) {
                    F4 v = load4(scan + (i * kWarps + seg) * kScanPad + lane * kV);
#pragma unroll
                    for (int j = 0; j < kV; ++j) m[j].set(i, v.v[j]);
                }
#pragma unroll
                for (int j = 0; j < kV; ++j) ex[j] = compose(m[j], ex[j]);
            }

            // 4. Decoupled look-back across CTAs (warp 0, lane owns 4 channels)
            if (w == 0) {
                float yin[NS][kV];
                const bool ok = lookback<Map, NS>(ticket, BS, c > 0, k, ex, init, yin, p.desc, lane, err,
                                                  p.wait_ns);
#pragma unroll
                for (int q = 0; q < NS; ++q) store4(scarry + q * kDc + lane * kV, yin[q]);
                if (lane == 0) s_int[5] = ok ? 0 : 1;
#pragma unroll
                for (int j = 0; j < kV; ++j) ex[j] = Map::identity();  // warp 0's own prefix
            }
            __syncthreads();
            if (s_int[5]) break;  // a wait gave up (error raised): stop this pass

            // 5. Sweep 2: s^{k+1}_l = J_l s^{k+1}_{l-1} + o_l, write it, and the
            //    residual of the updated states F_l(H^{k+1}) for the convergence test
            {
                float2 y[NS][2];  // s^{k+1} at the row before the current one
#pragma unroll
                for (int j = 0; j < kV; ++j) {
                    float x[NS], z[NS];
#pragma unroll
                    for (int q = 0; q < NS; ++q) x[q] = scarry[q * kDc + lane * kV + j];
                    apply(ex[j], x, z);
#pragma unroll
                    for (int q = 0; q < NS; ++q) {
                        if (j & 1) y[q][j >> 1].y = z[q];
                        else y[q][j >> 1].x = z[q];
                    }
                }
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    const int row = r0 + t;
                    const long long l = l0 + row;
                    const bool lv = l < L;
                    float2 u[G][2];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        F4 x = load4(su + (row * G + g) * kDc + lane * kV);
                        u[g][0] = make_float2(x.v[0], x.v[1]);
                        u[g][1] = make_float2(x.v[2], x.v[3]);
                    }
                    float2 off[NS][2], sn[NS][2];
#pragma unroll
                    for (int q = 0; q < NS; ++q) {
                        const float* src =
                            (t == T - 1) ? slast + (q * kWarps + w) * kDc : ss + (q * Lc + row) * kDc;
                        F4 x = load4(src + lane * kV);
                        off[q][0] = make_float2(x.v[0], x.v[1]);
                        off[q][1] = make_float2(x.v[2], x.v[3]);
                    }
#pragma unroll
                    for (int jp = 0; jp < 2; ++jp) {
                        float2 yv[NS], uu[G], aa[G], f2[NS], jy[NS];
#pragma unroll
                        for (int q = 0; q < NS; ++q) yv[q] = y[q][jp];
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            uu[g] = u[g][jp];
                            aa[g] = wv[g][jp];
                        }
                        apply_matrix2(Jr[t][jp], yv, jy);
#pragma unroll
                        for (int q = 0; q < NS; ++q) sn[q][jp] = add2(jy[q], off[q][jp]);
                        Packed::value(yv, uu, aa, f2);
                        if (lv && chv) {
#pragma unroll
                            for (int q = 0; q < NS; ++q)
                                rpost = max(rpost, max(abs_bits(sn[q][jp].x - f2[q].x), abs_bits(sn[q][jp].y - f2[q].y)));
                        }
#pragma unroll
                        for (int q = 0; q < NS; ++q) y[q][jp] = sn[q][jp];
                    }
                    if (lv && chv) {
#pragma unroll
                        for (int q = 0; q < NS; ++q)
                            __stcg(reinterpret_cast<float4*>(p.st[q] + ((b * L + l) * D + dch)),
                                   make_float4(sn[q][0].x, sn[q][0].y, sn[q][1].x, sn[q][1].y));
                    }
                    if (row == Lc - 1 && c + 1 < p.n_chunks && chv) {
#pragma unroll
                        for (int q = 0; q < NS; ++q)
                            __stcg(reinterpret_cast<float4*>(
                                       p.bnd + ((((size_t)((k + 1) & 1) * NS + q) * p.B + b) * p.n_chunks + c) *
                                                   Dpad + dch),
                                   make_float4(sn[q][0].x, sn[q][0].y, sn[q][1].x, sn[q][1].y));
                    }
                }
            }
            // release the stage: every lane of this warp is done with it
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            stage ^= 1;
        }
        // The other stage holds one more completed phase (the prefetch past the
        // last tile, or a real tile if this pass stopped on an error): consume it.
        (void)mbar_wait_bounded(&full[stage ^ 1], (full_par >> (stage ^ 1)) & 1u, err, p.wait_ns);
        full_par ^= 1u << (stage ^ 1);
        // residual maxima of this CTA for this pass
        {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                rpost = max(rpost, __shfl_xor_sync(0xffffffffu, rpost, off));
                rpre = max(rpre, __shfl_xor_sync(0xffffffffu, rpre, off));
            }
            if (lane == 0) {
                s_red[w] = rpost;
                s_red[kWarps + w] = rpre;
            }
            __syncthreads();
            if (tid == 0) {
                unsigned a = 0u, b2 = 0u;
                for (int i = 0; i < kWarps; ++i) {
                    a = max(a, s_red[i]);
                    b2 = max(b2, s_red[kWarps + i]);
                }
                atomicMax(&hdr->res[slot], a);
                if (first) atomicMax(&hdr->res0, b2);
            }
        }

        const bool bar_ok = grid_barrier(&hdr->bar, unsigned(k), err, p.wait_ns, &s_int[2]);

        if (tid == 0) {
            NewtonDecision d = newton_decide(hdr, k, slot, bar_ok, p.tol, p.max_iters);
            if (!d.cont && blockIdx.x == 0) newton_publish(hdr, d, k);
            s_int[3] = d.cont;
            s_int[4] = d.zero;
        }
        __syncthreads();
        if (!s_int[3]) {
            if (s_int[4]) newton_zero_states<NS>(p, tid, blockDim.x);
            return;
        }
        if (tid == 0) fence_proxy_async_global();  // other CTAs' state writes before our next TMA reads
    }
}

}  // namespace pararnn
