// Adjoint (reverse-time) scan for training gradients through the Newton
// solution of a ParaGRU / ParaLSTM recurrence.
//
// The pages ("ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e
// escala pra 7B parâmetros") describe the forward solve only.  The reading
// used here: at the solution F(H) = 0 the gradient of a loss with respect to
// the inputs is (dF/du)^T lambda where lambda solves the transposed Newton
// system, i.e. the reverse-time linear recurrence
//   lambda_l = g_l + J_{l+1}^T lambda_{l+1},   g_l = dLoss/dstate_l,
// again a linear SSM (section "A sacada: método de Newton"), with the same
// diagonal / 2x2 structure (section "Engenharia pra escalar").  It is scanned
// with the same three-level machinery as the forward solve, in reverse:
// with mu_l = J_l^T lambda_l each step is the affine map
//   mu_l = J_l^T mu_{l+1} + J_l^T g_l,
// whose maps depend only on step l's own data.  Then lambda_l = g_l + mu_{l+1},
// du_l follows from lambda_l by the chain rule of the cell, da sums
// (d pre / d a) du over b and l in a fixed order (deterministic), and the
// gradient of the initial state is mu_1.
#pragma once

#include <climits>

#include "scan_common.cuh"

namespace pararnn {

struct AdjointParams {
    const float* a;       // [G][D]
    const float* s0[2];   // initial state per component [B][D] (NULL = zeros)
    const float* st[2];   // forward states per component [B][L][D]
    float* du;            // [B][L][G][D]
    float* ds0[2];        // gradient of the initial state per component [B][D] (NULL = not wanted)
    long long B, L, D;
    int S, n_chunks, n_tiles;
    int has_g[2];         // upstream gradient present per state component
    WsHeader* hdr;
    unsigned long long* desc;  // [n_tiles][desc_words] tagged words
    float* partial;       // [B][n_chunks][S][G][kDc] per-tile sums for da
    unsigned long long wait_ns;
};

template <class Cell, class UT, int T>
struct AdjointLayout {
    static constexpr int G = Cell::G;
    static constexpr int NS = Cell::NS;
    static constexpr int NC = Cell::Map::kFloats;
    static constexpr int Lc = kWarps * T;
    static constexpr size_t u_bytes = size_t(Lc) * G * kDc * sizeof(UT);
    static constexpr size_t s_bytes = size_t(Lc) * kDc * sizeof(float);
    static constexpr size_t scan_floats = size_t(NC) * kWarps * kScanPad;
    static constexpr size_t red_floats = size_t(kWarps) * G * kDc;
    // stage: gates | states [NS][Lc][kDc] | upstream [NS][Lc][kDc]
    static constexpr size_t off_u = 0;
    static constexpr size_t off_s = off_u + u_bytes;
    static constexpr size_t off_g = off_s + NS * s_bytes;
    static constexpr size_t stage_bytes = off_g + NS * s_bytes;
    // after the stages: scan scratch (reused for the da reduction), tile
    // aggregate, carry, two mbarriers and the stages' tickets
    static constexpr size_t rest_bytes = 4 * (scan_floats > red_floats ? scan_floats : red_floats) +
                                         size_t(NC) * kDc * 4 + size_t(NS) * kDc * 4 + 64;
    // two stages (the next tile loads while this one is swept) where they fit
    static constexpr int kStg = 2 * stage_bytes + rest_bytes <= 232448 ? 2 : 1;
    static constexpr size_t off_scan = kStg * stage_bytes;
    static constexpr size_t off_tagg = off_scan + 4 * (scan_floats > red_floats ? scan_floats : red_floats);
    static constexpr size_t off_carry = off_tagg + size_t(NC) * kDc * 4;
    static constexpr size_t off_misc = off_carry + size_t(NS) * kDc * 4;
    static constexpr size_t smem_bytes = off_misc + 64;
    static constexpr int desc_words = TileDesc<typename Cell::Map, NS>::words;
    static_assert(smem_bytes <= 232448, "shared memory");
};

template <class Cell, class UT, int T>
__global__ void __launch_bounds__(kThreads, 1)
    adjoint_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_s0,
                   const __grid_constant__ CUtensorMap tm_s1, const __grid_constant__ CUtensorMap tm_g0,
                   const __grid_constant__ CUtensorMap tm_g1, const AdjointParams p)
{
    using LY = AdjointLayout<Cell, UT, T>;
    using Map = typename Cell::Map;
    constexpr int G = LY::G, NS = LY::NS, NC = LY::NC, Lc = LY::Lc;

    constexpr int NSTG = LY::kStg;
    extern __shared__ __align__(128) unsigned char smem[];
    float* scan = reinterpret_cast<float*>(smem + LY::off_scan);
    float* tagg = reinterpret_cast<float*>(smem + LY::off_tagg);
    float* scarry = reinterpret_cast<float*>(smem + LY::off_carry);
    uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + LY::off_misc);  // [NSTG]
    int* s_int = reinterpret_cast<int*>(smem + LY::off_misc + 16);      // [0..1] flags, [2..3] tickets

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    WsHeader* hdr = p.hdr;
    int* err = &hdr->error;
    const long long D = p.D, L = p.L;
    const int BS = int(p.B) * p.S;

    // thread 0: ticket t's loads into stage i (no-op for an invalid ticket)
    auto issue = [&](int t, int i) {
        s_int[2 + i] = t;
        if (t >= p.n_tiles) return;
        const int cc = p.n_chunks - 1 - t / BS, rr = t % BS;
        const int bb = rr / p.S, dd = (rr - bb * p.S) * kDc, ll = cc * Lc;
        unsigned char* st = smem + i * LY::stage_bytes;
        fence_proxy_async_shared();
        uint32_t bytes = uint32_t(LY::u_bytes + NS * LY::s_bytes);
#pragma unroll
        for (int q = 0; q < NS; ++q)
            if (p.has_g[q]) bytes += uint32_t(LY::s_bytes);
        mbar_arrive_expect_tx(&mbar[i], bytes);
        tma_load_4d(st + LY::off_u, &tm_u, dd, 0, ll, bb, &mbar[i]);
        tma_load_3d(st + LY::off_s, &tm_s0, dd, ll, bb, &mbar[i]);
        if (NS == 2) tma_load_3d(st + LY::off_s + LY::s_bytes, &tm_s1, dd, ll, bb, &mbar[i]);
        if (p.has_g[0]) tma_load_3d(st + LY::off_g, &tm_g0, dd, ll, bb, &mbar[i]);
        if (NS == 2 && p.has_g[NS - 1]) tma_load_3d(st + LY::off_g + LY::s_bytes, &tm_g1, dd, ll, bb, &mbar[i]);
    };
    auto take = [&]() {
        const int t = int(atomicAdd(&hdr->tick[0], 1u));
        return error_raised(err) ? INT_MAX : t;
    };

    if (tid == 0) {
        for (int i = 0; i < NSTG; ++i) mbar_init(&mbar[i], 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_u);
        // tickets are taken in order and handled in order, tile n in stage n % NSTG
        for (int i = 0; i < NSTG; ++i) issue(take(), i);
    }
    __syncthreads();

    for (int n = 0;; ++n) {
        // the tile before this one is finished: its stage takes tile n+NSTG-1
        if (n >= 1 && tid == 0) {
            const int last = s_int[2 + (n - 1) % NSTG];
            issue(last < p.n_tiles ? take() : INT_MAX, (n + NSTG - 1) % NSTG);
        }
        __syncthreads();
        const int stg = n % NSTG;
        const int ticket = s_int[2 + stg];
        if (ticket >= p.n_tiles) break;
        UT* su = reinterpret_cast<UT*>(smem + stg * LY::stage_bytes + LY::off_u);
        float* ss = reinterpret_cast<float*>(smem + stg * LY::stage_bytes + LY::off_s);
        float* sg = reinterpret_cast<float*>(smem + stg * LY::stage_bytes + LY::off_g);
        // reverse chunk order: the last chunk gets the first tickets
        const int c = p.n_chunks - 1 - ticket / BS;
        const int rem = ticket % BS;
        const int b = rem / p.S;
        const int sl = rem - b * p.S;
        const int l0 = c * Lc;
        const int d0 = sl * kDc;

        const int dch = d0 + lane * kV;
        const bool chv = dch < D;
        float wv[G][kV];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            F4 x = chv ? load4(p.a + g * D + dch) : F4{{0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int j = 0; j < kV; ++j) wv[g][j] = x.v[j];
        }
        // state just before the chunk (forward states are read-only here)
        float halo[NS][kV];
#pragma unroll
        for (int q = 0; q < NS; ++q) {
            F4 x{{0.f, 0.f, 0.f, 0.f}};
            if (chv) {
                if (c == 0) {
                    if (p.s0[q]) x = load4(p.s0[q] + b * D + dch);
                } else {
                    x = load4(p.st[q] + ((b * L + l0 - 1) * D + dch));
                }
            }
#pragma unroll
            for (int j = 0; j < kV; ++j) halo[q][j] = x.v[j];
        }
        (void)mbar_wait_bounded(&mbar[stg], uint32_t(n / NSTG) & 1u, err, p.wait_ns);

        const int r0 = w * T;
        // element access helpers (row within the tile)
        auto prev_state = [&](int row, float (&sv)[NS][kV]) {
#pragma unroll
            for (int q = 0; q < NS; ++q) {
                if (row == 0) {
#pragma unroll
                    for (int j = 0; j < kV; ++j) sv[q][j] = halo[q][j];
                } else {
                    F4 x = load4(ss + (q * Lc + row - 1) * kDc + lane * kV);
#pragma unroll
                    for (int j = 0; j < kV; ++j) sv[q][j] = x.v[j];
                }
            }
        };
        auto upstream = [&](int row, float (&gv)[NS][kV]) {
#pragma unroll
            for (int q = 0; q < NS; ++q) {
                F4 x{{0.f, 0.f, 0.f, 0.f}};
                if (p.has_g[q]) x = load4(sg + (q * Lc + row) * kDc + lane * kV);
#pragma unroll
                for (int j = 0; j < kV; ++j) gv[q][j] = x.v[j];
            }
        };

        // Sweep 1 (reverse within the thread's rows): fold the maps
        Map agg[kV];
#pragma unroll
        for (int j = 0; j < kV; ++j) agg[j] = Map::identity();
#pragma unroll
        for (int t = T - 1; t >= 0; --t) {
            const int row = r0 + t;
            float sv[NS][kV], gv[NS][kV];
            prev_state(row, sv);
            upstream(row, gv);
            F4 ug[G];
#pragma unroll
            for (int g = 0; g < G; ++g) ug[g] = load4(su + (row * G + g) * kDc + lane * kV);
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
        // warp w's rows come after warp w+1's in the reverse scan order
        scan_put(scan, kWarps - 1 - w, lane, agg);
        __syncthreads();
        cta_segment_scan<Map>(scan, tagg, tid);
        __syncthreads();

        if (w == 0) {
            Map ta[kV];
#pragma unroll
            for (int i = 0; i < NC; ++i) {
                F4 v = load4(tagg + i * kDc + lane * kV);
#pragma unroll
                for (int j = 0; j < kV; ++j) ta[j].set(i, v.v[j]);
            }
            float zero[NS][kV], cr[NS][kV];
#pragma unroll
            for (int q = 0; q < NS; ++q)
#pragma unroll
                for (int j = 0; j < kV; ++j) zero[q][j] = 0.f;
            // mu_{L+1} = 0 enters the last chunk
            const bool ok = lookback<Map, NS>(ticket, BS, c < p.n_chunks - 1, 0, ta, zero, cr, p.desc, lane,
                                              err, p.wait_ns);
#pragma unroll
            for (int q = 0; q < NS; ++q) store4(scarry + q * kDc + lane * kV, cr[q]);
            if (lane == 0) s_int[1] = ok ? 0 : 1;
        }
        __syncthreads();
        if (s_int[1]) {
            // look-back gave up: let the next tile's copy land before leaving
            if (NSTG > 1 && tid == 0 && s_int[2 + (n + 1) % NSTG] < p.n_tiles)
                (void)mbar_wait_bounded(&mbar[(n + 1) % NSTG], uint32_t((n + 1) / NSTG) & 1u, err, p.wait_ns);
            break;
        }

        // Sweep 2 (reverse): lambda, du, da partials, mu
        float dacc[G][kV];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int j = 0; j < kV; ++j) dacc[g][j] = 0.f;
        float mu[NS][kV];
#pragma unroll
        for (int j = 0; j < kV; ++j) {
            Map ex = scan_get<Map>(scan, kWarps - 1 - w, lane * kV + j);
            float x[NS], y[NS];
#pragma unroll
            for (int q = 0; q < NS; ++q) x[q] = scarry[q * kDc + lane * kV + j];
            apply(ex, x, y);
#pragma unroll
            for (int q = 0; q < NS; ++q) mu[q][j] = y[q];
        }
#pragma unroll
        for (int t = T - 1; t >= 0; --t) {
            const int row = r0 + t;
            const long long l = l0 + row;
            const bool lv = l < L;
            float sv[NS][kV], gv[NS][kV];
            prev_state(row, sv);
            upstream(row, gv);
            F4 ug[G];
#pragma unroll
            for (int g = 0; g < G; ++g) ug[g] = load4(su + (row * G + g) * kDc + lane * kV);
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
                    aa[g] = wv[g][j];
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
                for (int g = 0; g < G; ++g) store4(p.du + (((b * L + l) * G + g) * D + dch), duv[g]);
            }
            if (l == 0 && chv) {
#pragma unroll
                for (int q = 0; q < NS; ++q)
                    if (p.ds0[q]) store4(p.ds0[q] + b * D + dch, mu[q]);
            }
        }
        // da: sum the 8 warps' partials in a fixed order
        __syncthreads();  // scan scratch is reused below
        float* red = scan;  // [kWarps][G][kDc]
#pragma unroll
        for (int g = 0; g < G; ++g) store4(red + (w * G + g) * kDc + lane * kV, dacc[g]);
        __syncthreads();
        float* part = p.partial + (((size_t)b * p.n_chunks + c) * p.S + sl) * G * kDc;
        for (int i = tid; i < G * kDc; i += kThreads) {
            float acc = 0.f;
#pragma unroll
            for (int ww = 0; ww < kWarps; ++ww) acc += red[ww * G * kDc + i];
            part[i] = acc;
        }
        __syncthreads();
    }
}

// da[g][d] = sum over b, then chunk c, of the per-tile partial sums, in a
// fixed order.  Block: 32 columns x 8 row-groups; each row-group sums every
// 8th (b, c) row, the 8 group sums are then added in group order.
__global__ void __launch_bounds__(256) da_reduce_kernel(const float* __restrict__ partial, float* __restrict__ da,
                                                        int rows /* B*n_chunks */, int S, int G, long long D)
{
    __shared__ float red[8][33];
    const int col = blockIdx.x * 32 + (threadIdx.x & 31);  // index over G*D
    const int grp = threadIdx.x >> 5;
    const long long GD = (long long)G * D;
    float acc = 0.f;
    int g = 0, s = 0, dd = 0;
    if (col < GD) {
        g = int(col / D);
        const long long d = col - (long long)g * D;
        s = int(d / kDc);
        dd = int(d - (long long)s * kDc);
        for (int r = grp; r < rows; r += 8) acc += partial[(((size_t)r * S + s) * G + g) * kDc + dd];
    }
    red[grp][threadIdx.x & 31] = acc;
    __syncthreads();
    if (grp == 0 && col < GD) {
        float t = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) t += red[i][threadIdx.x];
        da[col] = t;
    }
}

// ------------------------------------------------------------ self tests
// Each runs one of the bounded waits against a condition nothing satisfies.

// The look-back of tile 1 whose predecessor (tile 0) never publishes.
__global__ void selftest_lookback_kernel(unsigned long long* desc, int* err, unsigned long long limit_ns)
{
    Aff<1> ta[kV];
    float init[1][kV], carry[1][kV];
#pragma unroll
    for (int j = 0; j < kV; ++j) {
        ta[j] = Aff<1>::identity();
        init[0][j] = 0.f;
    }
    (void)lookback<Aff<1>, 1>(1, 1, true, 0, ta, init, carry, desc, threadIdx.x & 31, err, limit_ns);
}

__global__ void selftest_barrier_kernel(unsigned* counter, int* err, unsigned long long limit_ns)
{
    __shared__ int s_flag;
    if (blockIdx.x == gridDim.x - 1) return;  // this CTA never arrives
    (void)grid_barrier(counter, 0u, err, limit_ns, &s_flag);
}

}  // namespace pararnn
