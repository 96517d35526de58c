// Plain diagonal linear scan: one pass of the chunked parallel scan over the
// linear recurrence of the zero-weight GRU,
//   h_l = (1 - s(u_z,l)) h_{l-1} + s(u_z,l) tanh(u_c,l),
// reading two of the three gate streams.  It is the linear SSM of the page
// "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala pra
// 7B parâmetros" (section "O compromisso que SSMs fizeram") and serves as the
// lower bound of one scan pass for the same [B][L][3][D] input: a Newton
// iteration cannot move fewer bytes than this.
#pragma once

#include <climits>

#include "scan_common.cuh"

namespace pararnn {

struct LinScanParams {
    const float* h0;  // [B][D] or NULL
    float* h;         // [B][L][D]
    long long B, L, D;
    int S, n_chunks, n_tiles;
    WsHeader* hdr;
    unsigned long long* desc;  // [n_tiles][desc_words] tagged words
    unsigned long long wait_ns;
};

template <class UT, int T>
struct LinScanLayout {
    static constexpr int Lc = kWarps * T;
    static constexpr size_t g_bytes = size_t(Lc) * kDc * sizeof(UT);  // one gate stream
    static constexpr size_t stage_bytes = 2 * g_bytes;                 // gates z and c
    static constexpr size_t off_scan = 2 * stage_bytes;                // two pipeline stages
    static constexpr size_t off_tagg = off_scan + size_t(2) * kWarps * kScanPad * 4;
    static constexpr size_t off_carry = off_tagg + size_t(2) * kDc * 4;
    static constexpr size_t off_misc = off_carry + size_t(kDc) * 4;
    static constexpr size_t smem_bytes = off_misc + 64;
    static constexpr int desc_words = TileDesc<Aff<1>, 1>::words;
    static_assert(smem_bytes <= 232448, "shared memory");
};

__device__ __forceinline__ Aff<1> linear_gru_map(float uz, float uc)
{
    float z, t;
    sigmoid_tanh(uz, uc, z, t);
    return {1.0f - z, z * t};
}

template <class UT, int T>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
    linear_scan_kernel(const __grid_constant__ CUtensorMap tm_u1, const LinScanParams p)
{
    using LY = LinScanLayout<UT, T>;
    using Map = Aff<1>;
    constexpr int Lc = LY::Lc;
    extern __shared__ __align__(128) unsigned char smem[];
    float* scan = reinterpret_cast<float*>(smem + LY::off_scan);
    float* tagg = reinterpret_cast<float*>(smem + LY::off_tagg);
    float* scarry = reinterpret_cast<float*>(smem + LY::off_carry);
    uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + LY::off_misc);
    int* s_int = reinterpret_cast<int*>(smem + LY::off_misc + 16);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    int* err = &p.hdr->error;
    const long long D = p.D, L = p.L;
    const int BS = int(p.B) * p.S;
    if (tid == 0) {
        mbar_init(&mbar[0], 1);
        mbar_init(&mbar[1], 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_u1);
    }
    __syncthreads();
    uint32_t phases = 0;

    // thread 0: start the loads of tile t into `stage`
    auto load_tile = [&](int t, int stage) -> int {
        if (error_raised(err)) t = INT_MAX;
        if (t < p.n_tiles) {
            const int c = t / BS, rem = t - (t / BS) * BS;
            const int b = rem / p.S, d0 = (rem - b * p.S) * kDc;
            unsigned char* st = smem + stage * LY::stage_bytes;
            fence_proxy_async_shared();
            mbar_arrive_expect_tx(&mbar[stage], uint32_t(LY::stage_bytes));
            tma_load_4d(st, &tm_u1, d0, 0, c * Lc, b, &mbar[stage]);               // gate z
            tma_load_4d(st + LY::g_bytes, &tm_u1, d0, 2, c * Lc, b, &mbar[stage]);  // gate c
        }
        return t;
    };

    // tickets run one tile ahead of the loads, the loads one tile ahead of the compute
    int tnext = 0;
    if (tid == 0) {
        s_int[6] = load_tile(int(atomicAdd(&p.hdr->tick[0], 1u)), 0);
        tnext = int(atomicAdd(&p.hdr->tick[0], 1u));
    }
    __syncthreads();
    int ticket = s_int[6];
    int stage = 0;
    while (ticket < p.n_tiles) {
        if (tid == 0) {
            s_int[6 + (stage ^ 1)] = load_tile(tnext, stage ^ 1);
            tnext = int(atomicAdd(&p.hdr->tick[0], 1u));
        }
        const UT* sz = reinterpret_cast<const UT*>(smem + stage * LY::stage_bytes);
        const UT* sc = sz + Lc * kDc;
        const int c = ticket / BS;
        const int rem = ticket - c * BS;
        const int b = rem / p.S;
        const int sl = rem - b * p.S;
        const int l0 = c * Lc, d0 = sl * kDc;
        const int dch = d0 + lane * kV;
        const bool chv = dch < D;
        float init[1][kV];
        {
            F4 x{{0.f, 0.f, 0.f, 0.f}};
            if (chv && c == 0 && p.h0) x = load4(p.h0 + b * D + dch);
#pragma unroll
            for (int j = 0; j < kV; ++j) init[0][j] = x.v[j];
        }
        (void)mbar_wait_bounded(&mbar[stage], (phases >> stage) & 1u, err, p.wait_ns);
        phases ^= 1u << stage;

        const int r0 = w * T;
        // the step maps stay in registers for the second sweep
        Map agg[kV], mt[T][kV];
#pragma unroll
        for (int j = 0; j < kV; ++j) agg[j] = Map::identity();
#pragma unroll
        for (int t = 0; t < T; ++t) {
            const int row = r0 + t;
            F4 z4 = load4(sz + row * kDc + lane * kV), c4 = load4(sc + row * kDc + lane * kV);
#pragma unroll
            for (int j = 0; j < kV; ++j) {
                mt[t][j] = linear_gru_map(z4.v[j], c4.v[j]);
                agg[j] = compose(mt[t][j], agg[j]);
            }
        }
        scan_put(scan, w, lane, agg);
        __syncthreads();
        cta_segment_scan<Map>(scan, tagg, tid);
        __syncthreads();
        if (w == 0) {
            Map ta[kV];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                F4 v = load4(tagg + i * kDc + lane * kV);
#pragma unroll
                for (int j = 0; j < kV; ++j) ta[j].set(i, v.v[j]);
            }
            float cr[1][kV];
            const bool ok = lookback<Map, 1>(ticket, BS, c > 0, 0, ta, init, cr, p.desc, lane, err, p.wait_ns);
            store4(scarry + lane * kV, cr[0]);
            if (lane == 0) s_int[1] = ok ? 0 : 1;
        }
        __syncthreads();
        if (s_int[1]) {
            if (s_int[6 + (stage ^ 1)] < p.n_tiles)
                (void)mbar_wait_bounded(&mbar[stage ^ 1], (phases >> (stage ^ 1)) & 1u, err, p.wait_ns);
            break;
        }
        float hv[kV];
#pragma unroll
        for (int j = 0; j < kV; ++j) {
            Map ex = scan_get<Map>(scan, w, lane * kV + j);
            float x = scarry[lane * kV + j], y;
            apply(ex, &x, &y);
            hv[j] = y;
        }
#pragma unroll
        for (int t = 0; t < T; ++t) {
            const int row = r0 + t;
            const long long l = l0 + row;
#pragma unroll
            for (int j = 0; j < kV; ++j) hv[j] = fmaf(mt[t][j].m, hv[j], mt[t][j].v);
            if (l < L && chv) stcgv<kV>(p.h + ((b * L + l) * D + dch), hv);
        }
        __syncthreads();
        ticket = s_int[6 + (stage ^ 1)];
        stage ^= 1;
    }
}

}  // namespace pararnn
