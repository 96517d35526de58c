// Input projection fused with the first Newton pass (ParaGRU).
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros" -- "O compromisso que SSMs fizeram": the recurrence takes
// the input through a projection (B_l x_l) before the nonlinearity; "A sacada:
// método de Newton": the first Newton iteration linearises every step at the
// initial guess H^0 = 0, where the step maps depend on the gates alone.
//
// One CTA per tile of 128 timesteps x 64 channels of one batch row.  The gate
// pre-activations of the tile, u = x W^T + bias for the G gates of its 64
// channels (an M=128, N=64G, K=Din product), are computed on the tensor cores:
// TMA brings 64-wide K slices of x and W (128-byte swizzle) into a two-stage
// shared-memory ring, one thread issues tcgen05.mma (bf16 in, fp32
// accumulator in tensor memory), and tcgen05.commit releases each stage.  The
// epilogue then reads the accumulator from tensor memory (one timestep per
// thread), adds the bias, rounds to bf16 and writes u for the later passes,
// and runs Newton pass 0 on the tile: the step maps at H^0, their fold per
// quarter of the tile, a decoupled look-back along the sequence, the new
// states H^1, the residuals of H^0 and H^1.  The fused solve continues from
// H^1 with pass 1.
#pragma once

#include <climits>

#include "cells.cuh"
#include "scan_common.cuh"

namespace pararnn {

constexpr int kPM = 128;  // timesteps of a tile (accumulator rows, TMEM lanes)
constexpr int kPC = 64;   // channels of a tile
constexpr int kPK = 64;   // K slice of one stage (128 bytes of bf16)
constexpr int kPStages = 2;

// ------------------------------------------------------ tcgen05 wrappers
// (PTX ISA, tensor core 5th generation: tcgen05.alloc / mma / commit / ld.)

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major, kind::f16 (bf16 inputs)
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          bool accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// arrive on `bar` once every tcgen05.mma this thread issued so far is done
__device__ __forceinline__ void umma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// 8 consecutive fp32 columns of this warp's 32 TMEM lanes (one per thread)
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8])
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand tile written by TMA
// with the 128-byte swizzle: rows of 128 bytes, groups of 8 rows 1024 bytes
// apart (stride byte offset), the leading byte offset unused (1), the
// descriptor version of this architecture (1), swizzle mode 2 (128 B).
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* tile)
{
    const uint64_t addr = smem_addr(tile);
    return ((addr & 0x3FFFFull) >> 4) | (1ull << 16) | ((1024ull >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N and M as given.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// bf16 bits of x rounded to nearest even
__device__ __forceinline__ uint16_t bf16_bits_rn(float x)
{
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}

// ------------------------------------------------------------ the kernel

struct ProjectParams {
    const float* bias;  // [G][D] or NULL
    const float* a;     // [G][D] recurrence weights
    const float* h0;    // [B][D] or NULL
    uint16_t* u;        // [B][L][G][D] bf16 out
    float* h;           // [B][L][D] out: H^1
    long long B, L, D, Din;
    int Sf, n_chunks, n_tiles;  // channel blocks of kPC, chunks of kPM, tiles
    WsHeader* hdr;
    unsigned long long* desc;   // [n_tiles][kPDescWords] tagged words
    unsigned long long wait_ns;
};

template <int G>
struct ProjectLayout {
    static constexpr size_t a_bytes = size_t(kPM) * kPK * 2;        // 16 KB
    static constexpr size_t b_bytes = size_t(G) * kPC * kPK * 2;    // 8 KB per gate
    static constexpr size_t stage_bytes = a_bytes + b_bytes;
    static constexpr size_t ring_bytes = kPStages * stage_bytes;
    // after the main loop the ring holds the rounded gates, [kPM][su_row]
    static constexpr int su_row = G * kPC * 2 + 16;                 // bytes per timestep (padded)
    static_assert(size_t(kPM) * su_row <= ring_bytes, "gate tile fits the ring");
    static constexpr size_t off_misc = ring_bytes;
    // misc: full[S], empty[S], done barriers; TMEM address; flags;
    // quarter folds [4][kPC][2]; carry [kPC]; bias [G][kPC]; maxima [2][4]
    static constexpr size_t off_bar = off_misc;
    static constexpr size_t off_tmem = off_bar + (2 * kPStages + 1) * 8;
    static constexpr size_t off_flag = off_tmem + 8;
    static constexpr size_t off_qagg = off_flag + 24;
    static constexpr size_t off_carry = off_qagg + 4 * kPC * 2 * 4;
    static constexpr size_t off_bias = off_carry + kPC * 4;
    static constexpr size_t off_red = off_bias + G * kPC * 4;
    static constexpr size_t used = off_red + 2 * 4 * 4;
    static constexpr size_t smem_bytes = used + 1024;               // room to align the ring to 1024 B
};

// Look-back descriptor of a fused tile: [32 lanes][2 channels][m, v] then
// [32 lanes][2 channels][state], tagged words (tag 1: aggregate, 2: inclusive).
constexpr int kPDescAgg = 32 * 4;
constexpr int kPDescWords = 32 * 4 + 32 * 2;

__global__ void __launch_bounds__(128, 2)
    project_pass0_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                         const ProjectParams p)
{
    using Cell = GruCell;
    using Map = Aff<1>;
    constexpr int G = Cell::G;
    using LY = ProjectLayout<G>;
    constexpr int N = G * kPC;
    constexpr uint32_t kIdesc = idesc_bf16(kPM, N);

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + LY::off_bar);
    uint64_t* empty = full + kPStages;
    uint64_t* done = empty + kPStages;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + LY::off_tmem);
    int* s_flag = reinterpret_cast<int*>(smem + LY::off_flag);  // [0] ticket, [1] look-back failed
    float* qagg = reinterpret_cast<float*>(smem + LY::off_qagg);  // [4][kPC][2]
    float* scarry = reinterpret_cast<float*>(smem + LY::off_carry);
    float* sbias = reinterpret_cast<float*>(smem + LY::off_bias);
    float* sred = reinterpret_cast<float*>(smem + LY::off_red);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    WsHeader* hdr = p.hdr;
    int* err = &hdr->error;
    const long long L = p.L, D = p.D;
    const int BSf = int(p.B) * p.Sf;

    if (tid == 0) {
        const int t = int(atomicAdd(&hdr->tick[3], 1u));
        s_flag[0] = t;
        s_flag[1] = 0;
        if (t == 0) hdr->t_pass[0] = global_timer_ns();
        for (int i = 0; i < kPStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_w);
    }
    if (w == 0) {
        tmem_alloc(s_tmem, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int ticket = s_flag[0];
    const int mc = ticket / BSf, rem = ticket - (ticket / BSf) * BSf;
    const int b = rem / p.Sf, d0 = (rem - b * p.Sf) * kPC;
    const long long l0 = (long long)mc * kPM;
    for (int i = tid; i < G * kPC; i += 128) {
        const int g = i / kPC, c = i - g * kPC;
        sbias[i] = (p.bias && d0 + c < D) ? p.bias[g * D + d0 + c] : 0.f;
    }

    // ---------------------------------------------------- main loop (GEMM)
    const int nk = int((p.Din + kPK - 1) / kPK);
    if (w == 0 && lane == 0) {
        // producer: K slices of x (rows l0.., batch b) and of W (rows d0.. of each gate)
        for (int kc = 0; kc < nk; ++kc) {
            const int s = kc % kPStages;
            if (kc >= kPStages && !mbar_wait_bounded(&empty[s], uint32_t((kc / kPStages) - 1) & 1u, err, p.wait_ns))
                break;
            unsigned char* st = smem + s * LY::stage_bytes;
            mbar_arrive_expect_tx(&full[s], uint32_t(LY::stage_bytes));
            tma_load_3d(st, &tm_x, kc * kPK, int(l0), b, &full[s]);
#pragma unroll
            for (int g = 0; g < G; ++g)
                tma_load_3d(st + LY::a_bytes + g * (kPC * kPK * 2), &tm_w, kc * kPK, d0, g, &full[s]);
        }
    } else if (w == 1 && lane == 0) {
        // MMA issuer: four K=16 steps per slice (32 bytes apart inside the swizzle atom)
        for (int kc = 0; kc < nk; ++kc) {
            const int s = kc % kPStages;
            if (!mbar_wait_bounded(&full[s], uint32_t(kc / kPStages) & 1u, err, p.wait_ns)) break;
            tc_fence_after();
            const unsigned char* st = smem + s * LY::stage_bytes;
            const uint64_t ad = smem_desc_sw128(st), bd = smem_desc_sw128(st + LY::a_bytes);
#pragma unroll
            for (int kk = 0; kk < kPK / 16; ++kk)
                umma_bf16(tmem, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), kIdesc, (kc | kk) != 0);
            umma_commit(&empty[s]);  // the stage is free once these products are done
        }
        umma_commit(done);  // every product issued above is done
    }
    __syncwarp();
    const bool mma_ok = mbar_wait_bounded(done, 0u, err, p.wait_ns);
    tc_fence_after();
    __syncthreads();  // every TMA write of the ring has been consumed: the ring is free

    // ------------------------------------ epilogue 1: accumulator -> bf16 gates
    // thread t holds timestep l0 + t (TMEM lane t); rounded gates go to the
    // ring ([t][g][c] bf16, rows padded) and to u in global memory
    unsigned char* su = smem;
    {
        const int t = tid;
        const long long l = l0 + t;
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int cc = 0; cc < kPC / 8; ++cc) {
                float v[8];
                tmem_ld8(tmem + (uint32_t(32 * w) << 16) + uint32_t(g * kPC + 8 * cc), v);
                tmem_wait_ld();
                uint32_t pk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float x0 = mma_ok ? v[2 * i] + sbias[g * kPC + 8 * cc + 2 * i] : 0.f;
                    const float x1 = mma_ok ? v[2 * i + 1] + sbias[g * kPC + 8 * cc + 2 * i + 1] : 0.f;
                    pk[i] = uint32_t(bf16_bits_rn(x0)) | (uint32_t(bf16_bits_rn(x1)) << 16);
                }
                const uint4 q = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *reinterpret_cast<uint4*>(su + t * LY::su_row + (g * kPC + 8 * cc) * 2) = q;
                if (l < L && d0 + 8 * cc < D)
                    *reinterpret_cast<uint4*>(p.u + ((b * L + l) * G + g) * D + d0 + 8 * cc) = q;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tmem, 256);

    // ------------------------------------------ epilogue 2: Newton pass 0
    // warp w: timesteps 32w..32w+31 of the tile (a quarter); lane: channels
    // lane, lane+32
    constexpr int kQ = kPM / 4;
    const int r0 = kQ * w;
    float aw[2][G], hp[2];
    bool cv[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int c = lane + 32 * j;
        cv[j] = d0 + c < D;
#pragma unroll
        for (int g = 0; g < G; ++g) aw[j][g] = cv[j] ? p.a[g * D + d0 + c] : 0.f;
        hp[j] = (l0 == 0 && p.h0 && cv[j]) ? p.h0[b * D + d0 + c] : 0.f;  // state before step l0 at H^0
    }
    auto gate = [&](int r, int g, int c) {
        const uint16_t x = *reinterpret_cast<const uint16_t*>(su + r * LY::su_row + (g * kPC + c) * 2);
        return __uint_as_float(uint32_t(x) << 16);
    };
    float Jm[kQ][2], Ov[kQ][2];  // the step maps, kept for the second sweep
    float r0max = 0.f;
    Map qa[2] = {Map::identity(), Map::identity()};
#pragma unroll
    for (int i = 0; i < kQ; ++i) {
        const int r = r0 + i;
        const bool lv = l0 + r < L;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int c = lane + 32 * j;
            float uu[G], f[1], s[1] = {(r == 0) ? hp[j] : 0.f};
#pragma unroll
            for (int g = 0; g < G; ++g) uu[g] = gate(r, g, c);
            Map m;
            Cell::eval(s, uu, aw[j], f, m);
            m.v = f[0] - m.m * s[0];
            if (!lv) m = Map::identity();  // steps beyond L leave the state as it is
            Jm[i][j] = m.m;
            Ov[i][j] = m.v;
            if (lv && cv[j]) r0max = max_keep_nan(r0max, fabsf(f[0]));  // F(H^0)_l = 0 - f
            qa[j] = compose(m, qa[j]);
        }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int c = lane + 32 * j;
        qagg[(w * kPC + c) * 2 + 0] = qa[j].m;
        qagg[(w * kPC + c) * 2 + 1] = qa[j].v;
    }
    __syncthreads();

    // warp 0: the tile's map per channel, the decoupled look-back, the carry
    if (w == 0) {
        const unsigned t_agg = 1u, t_incl = 2u;
        Map ta[2];
        float carry[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int c = lane + 32 * j;
            Map acc = Map::identity();
#pragma unroll
            for (int q = 0; q < 4; ++q) acc = compose(Map{qagg[(q * kPC + c) * 2], qagg[(q * kPC + c) * 2 + 1]}, acc);
            ta[j] = acc;
            carry[j] = (l0 == 0 && p.h0 && cv[j]) ? p.h0[b * D + d0 + c] : 0.f;
        }
        unsigned long long* mine = p.desc + (size_t)ticket * kPDescWords;
        bool ok = true;
        if (mc > 0) {
            st_words2(mine + lane * 4, tag_word(ta[0].m, t_agg), tag_word(ta[0].v, t_agg));
            st_words2(mine + lane * 4 + 2, tag_word(ta[1].m, t_agg), tag_word(ta[1].v, t_agg));
            Map acc[2] = {Map::identity(), Map::identity()};
            int jt = ticket - BSf;
            bool resolved = false;
            uint64_t t0 = 0;
            unsigned spins = 0;
            while (__any_sync(0xffffffffu, !resolved)) {
                if (!resolved) {
                    const unsigned long long* pd = p.desc + (size_t)jt * kPDescWords;
                    unsigned long long wi0, wi1, wa0, wa1, wa2, wa3;
                    ld_words2(pd + kPDescAgg + lane * 2, wi0, wi1);
                    ld_words2(pd + lane * 4, wa0, wa1);
                    ld_words2(pd + lane * 4 + 2, wa2, wa3);
                    if (unsigned(wi0 >> 32) == t_incl && unsigned(wi1 >> 32) == t_incl) {
                        carry[0] = fmaf(acc[0].m, __uint_as_float(unsigned(wi0)), acc[0].v);
                        carry[1] = fmaf(acc[1].m, __uint_as_float(unsigned(wi1)), acc[1].v);
                        resolved = true;
                    } else if (unsigned(wa0 >> 32) == t_agg && unsigned(wa1 >> 32) == t_agg &&
                               unsigned(wa2 >> 32) == t_agg && unsigned(wa3 >> 32) == t_agg) {
                        acc[0] = compose(acc[0], Map{__uint_as_float(unsigned(wa0)), __uint_as_float(unsigned(wa1))});
                        acc[1] = compose(acc[1], Map{__uint_as_float(unsigned(wa2)), __uint_as_float(unsigned(wa3))});
                        jt -= BSf;
                        spins = 0;
                    } else {
                        if ((++spins & 15u) == 0u) {
                            const uint64_t now = global_timer_ns();
                            if (error_raised(err)) {
                                ok = false;
                                resolved = true;
                            } else if (t0 == 0) {
                                t0 = now;
                            } else if (now - t0 > p.wait_ns) {
                                raise_error(err, PARARNN_ERR_TIMEOUT);
                                ok = false;
                                resolved = true;
                            }
                        }
                        if (spins > 32) __nanosleep(64);
                    }
                }
            }
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            float i0 = fmaf(ta[0].m, carry[0], ta[0].v), i1 = fmaf(ta[1].m, carry[1], ta[1].v);
            st_words2(mine + kPDescAgg + lane * 2, tag_word(i0, t_incl), tag_word(i1, t_incl));
        }
        scarry[lane] = carry[0];
        scarry[lane + 32] = carry[1];
        if (lane == 0) s_flag[1] = ok ? 0 : 1;
    }
    __syncthreads();

    // state entering this warp's quarter, then H^1 and the residual of H^1
    float r1max = 0.f;
    if (!s_flag[1]) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int c = lane + 32 * j;
            float y = scarry[c];
            for (int q = 0; q < w; ++q) y = fmaf(qagg[(q * kPC + c) * 2], y, qagg[(q * kPC + c) * 2 + 1]);
            float prev = y;  // H^1 before step r0
#pragma unroll
            for (int i = 0; i < kQ; ++i) {
                const int r = r0 + i;
                const long long l = l0 + r;
                const float hn = fmaf(Jm[i][j], prev, Ov[i][j]);
                if (l < L && cv[j]) {
                    float uu[G], f[1], s[1] = {prev};
#pragma unroll
                    for (int g = 0; g < G; ++g) uu[g] = gate(r, g, c);
                    Cell::value(s, uu, aw[j], f);
                    r1max = max_keep_nan(r1max, fabsf(hn - f[0]));
                    __stcg(p.h + (b * L + l) * D + d0 + c, hn);
                }
                prev = hn;
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        r0max = max_keep_nan(r0max, __shfl_xor_sync(0xffffffffu, r0max, off));
        r1max = max_keep_nan(r1max, __shfl_xor_sync(0xffffffffu, r1max, off));
    }
    if (lane == 0) {
        sred[w] = r0max;
        sred[4 + w] = r1max;
    }
    __syncthreads();
    if (tid == 0) {
        float x0 = 0.f, x1 = 0.f;
        for (int i = 0; i < 4; ++i) {
            x0 = max_keep_nan(x0, sred[i]);
            x1 = max_keep_nan(x1, sred[4 + i]);
        }
        atomicMax(&hdr->res0, __float_as_uint(x0) & 0x7fffffffu);
        atomicMax(&hdr->res[0], __float_as_uint(x1) & 0x7fffffffu);
        if (ticket == 0) hdr->k0 = 1;  // the fused solve continues with pass 1
    }
}

}  // namespace pararnn
