// Input projection fused with the first Newton pass (ParaGRU).
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros" -- "O compromisso que SSMs fizeram": the recurrence takes
// the input through a projection (B_l x_l) before the nonlinearity; "A sacada:
// método de Newton": the first Newton iteration linearises every step at the
// initial guess H^0 = 0, where the step maps depend on the gates alone.
//
// A tile is 128 timesteps x 64 channels of one batch row.  Its gate
// pre-activations, u = x W^T + bias for the G gates of its 64 channels (an
// M=128, N=64G, K=Din product), are computed on the tensor cores: a TMA warp
// brings 64-wide K slices of x and W (128-byte swizzle) into a four-stage
// shared-memory ring, one thread issues tcgen05.mma (bf16 in, fp32
// accumulator in tensor memory) and tcgen05.commit releases each stage.
// Sixteen epilogue warps read the accumulator (one timestep per thread), add
// the bias, round to bf16 into shared memory, write u for the later passes
// from there in whole 128-byte lines, and run Newton pass 0 on the tile: the step maps at H^0, their fold per quarter of the tile, a
// decoupled look-back along the sequence, the new states H^1 and the
// residuals of H^0 and H^1.  Two accumulators let the next tile's products
// run during this tile's epilogue.  The fused solve continues from H^1 with
// pass 1.
#pragma once

#include <climits>

#include "cells.cuh"
#include "scan_common.cuh"

namespace pararnn {

constexpr int kPM = 128;  // timesteps of a tile (accumulator rows, TMEM lanes)
constexpr int kPC = 64;   // channels of a tile
constexpr int kPK = 64;   // K slice of one stage (128 bytes of bf16)

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

// Warp roles of the persistent kernel: 0 loads (TMA), 1 issues the products,
// 2..17 run the epilogue.  Reading the accumulator, warp w takes TMEM lanes
// 32*(w % 4) (a quarter of the tile's timesteps) and a quarter of its columns;
// in the Newton pass, epilogue warp e takes timesteps 16*(e/2) .. +15 and
// channels 32*(e%2) .. +31, one per lane.
constexpr int kPEpiWarps = 16;
constexpr int kPThreads = 32 * (2 + kPEpiWarps);
constexpr int kPEpiBar = 1;  // named barrier of the epilogue warps
constexpr int kPRowGroups = kPEpiWarps / 2;  // row groups of the Newton pass

template <int G>
struct ProjectLayout {
    static constexpr int kStages = 4;
    static constexpr size_t a_bytes = size_t(kPM) * kPK * 2;        // 16 KB
    static constexpr size_t b_bytes = size_t(G) * kPC * kPK * 2;    // 8 KB per gate
    static constexpr size_t stage_bytes = a_bytes + b_bytes;
    static constexpr size_t ring_bytes = kStages * stage_bytes;
    // the rounded gates of the tile in the epilogue, by pairs of timesteps:
    // [kPM / 2][G][kPC] words, each holding the bf16 gate of timesteps 2i (low
    // half) and 2i + 1 (high half); rows padded so that the 16-byte writes of
    // eight consecutive timesteps fall in distinct banks
    static constexpr int su_row = G * kPC * 4 + 32;                 // bytes per pair of timesteps
    static constexpr size_t off_su = ring_bytes;
    static constexpr size_t off_misc = off_su + size_t(kPM / 2) * su_row;
    // misc: full[S], empty[S], tmem_full[2], tmem_empty[2]; TMEM address;
    // flags; row-group folds [kPRowGroups][kPC][2]; carry [kPC]; bias
    // [G][kPC]; maxima [2][kPEpiWarps]
    static constexpr size_t off_bar = off_misc;
    static constexpr size_t off_tmem = off_bar + (2 * kStages + 4) * 8;
    static constexpr size_t off_flag = off_tmem + 8;
    static constexpr size_t off_qagg = off_flag + 8;
    static constexpr size_t off_carry = off_qagg + kPRowGroups * kPC * 2 * 4;
    static constexpr size_t off_bias = off_carry + kPC * 4;
    static constexpr size_t off_red = off_bias + G * kPC * 4;
    static constexpr size_t used = off_red + 2 * kPEpiWarps * 4;
    static constexpr size_t smem_bytes = used + 1024;               // room to align the ring to 1024 B
    static_assert(smem_bytes <= 232448, "shared memory");
};

// Look-back descriptor of a fused tile: [32 lanes][2 channels][m, v] then
// [32 lanes][2 channels][state], tagged words (tag 1: aggregate, 2: inclusive).
constexpr int kPDescAgg = 32 * 4;
constexpr int kPDescWords = 32 * 4 + 32 * 2;

__device__ __forceinline__ void epi_sync()
{
    asm volatile("bar.sync %0, %1;" ::"n"(kPEpiBar), "n"(32 * kPEpiWarps) : "memory");
}

// One persistent CTA per SM, every CTA resident (cooperative launch).  CTA c
// takes tiles c, c + grid, c + 2 grid, ... in ticket order (chunk-major), so a
// tile's predecessor along its sequence has a smaller ticket and is handled
// by a resident CTA at the same or an earlier step: the look-backs cannot
// deadlock.  The loads and products of the next tile run while the epilogue
// of this one does (two accumulators in tensor memory).
__global__ void __launch_bounds__(kPThreads, 1)
    project_pass0_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                         const ProjectParams p)
{
    using Cell = GruCell;
    using Map = Aff<1>;
    constexpr int G = Cell::G;
    using LY = ProjectLayout<G>;
    constexpr int S = LY::kStages;
    constexpr int N = G * kPC;
    constexpr uint32_t kIdesc = idesc_bf16(kPM, N);
    constexpr uint32_t kAccCols = 256;  // one accumulator (N <= 256 columns)

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + LY::off_bar);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;   // [2] accumulator written
    uint64_t* tempty = tfull + 2;  // [2] accumulator read
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + LY::off_tmem);
    int* s_flag = reinterpret_cast<int*>(smem + LY::off_flag);    // [0] look-back failed
    float* qagg = reinterpret_cast<float*>(smem + LY::off_qagg);  // [kPRowGroups][kPC][2]
    float* scarry = reinterpret_cast<float*>(smem + LY::off_carry);
    float* sbias = reinterpret_cast<float*>(smem + LY::off_bias);
    float* sred = reinterpret_cast<float*>(smem + LY::off_red);
    unsigned char* su = smem + LY::off_su;

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    WsHeader* hdr = p.hdr;
    int* err = &hdr->error;
    const long long L = p.L, D = p.D;
    const int BSf = int(p.B) * p.Sf;
    const int nk = int((p.Din + kPK - 1) / kPK);
    const int n_mine = p.n_tiles > int(blockIdx.x) ? (p.n_tiles - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;

    if (tid == 0) {
        if (blockIdx.x == 0) hdr->t_pass[0] = global_timer_ns();
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], kPEpiWarps);  // one arrival per epilogue warp
        }
        fence_mbar_init();
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_w);
    }
    if (w == 0) {
        tmem_alloc(s_tmem, 2 * kAccCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (w == 0) {
        // ---------------------------------------------------------- loads
        if (lane == 0) {
            for (int st = 0; st < n_mine; ++st) {
                const int t = int(blockIdx.x) + st * int(gridDim.x);
                const int mc = t / BSf, rem = t - (t / BSf) * BSf;
                const int b = rem / p.Sf, d0 = (rem - b * p.Sf) * kPC;
                bool ok = true;
                for (int kc = 0; kc < nk; ++kc) {
                    const int q = st * nk + kc, s = q % S;
                    if (q >= S && !mbar_wait_bounded(&empty[s], uint32_t((q / S) - 1) & 1u, err, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    unsigned char* sp = smem + s * LY::stage_bytes;
                    mbar_arrive_expect_tx(&full[s], uint32_t(LY::stage_bytes));
                    tma_load_3d(sp, &tm_x, kc * kPK, mc * kPM, b, &full[s]);
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        tma_load_3d(sp + LY::a_bytes + g * (kPC * kPK * 2), &tm_w, kc * kPK, d0, g, &full[s]);
                }
                if (!ok) break;
            }
        }
    } else if (w == 1) {
        // ------------------------------------------------------- products
        if (lane == 0) {
            for (int st = 0; st < n_mine; ++st) {
                const int acc = st & 1;
                if (st >= 2 && !mbar_wait_bounded(&tempty[acc], uint32_t((st / 2) - 1) & 1u, err, p.wait_ns)) break;
                tc_fence_after();
                const uint32_t td = tmem + uint32_t(acc) * kAccCols;
                bool ok = true;
                for (int kc = 0; kc < nk; ++kc) {
                    const int q = st * nk + kc, s = q % S;
                    if (!mbar_wait_bounded(&full[s], uint32_t(q / S) & 1u, err, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const unsigned char* sp = smem + s * LY::stage_bytes;
                    const uint64_t ad = smem_desc_sw128(sp), bd = smem_desc_sw128(sp + LY::a_bytes);
                    // four K=16 steps, 32 bytes apart inside the swizzle atom
#pragma unroll
                    for (int kk = 0; kk < kPK / 16; ++kk)
                        umma_bf16(td, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), kIdesc, (kc | kk) != 0);
                    umma_commit(&empty[s]);  // the stage is free once these products are done
                }
                umma_commit(&tfull[acc]);  // the accumulator is complete
                if (!ok) break;
            }
        }
    } else {
        // ------------------------------------------------------- epilogue
        const int e = w - 2;                  // epilogue warp 0..15
        const int et = tid - 64;              // 0..511 among the epilogue threads
        const int lq = w & 3;                 // TMEM lane quarter this warp can read
        const int cq = e >> 2;                // its quarter of the accumulator columns
        constexpr int kRows = kPM / kPRowGroups;  // timesteps of a row group (16)
        const int rg = e >> 1;                // Newton pass: row group
        const int c = 32 * (e & 1) + lane;    // and channel
        const int r0 = kRows * rg;
        for (int st = 0; st < n_mine; ++st) {
            const int t = int(blockIdx.x) + st * int(gridDim.x);
            const int mc = t / BSf, rem = t - (t / BSf) * BSf;
            const int b = rem / p.Sf, d0 = (rem - b * p.Sf) * kPC;
            const long long l0 = (long long)mc * kPM;
            const int acc = st & 1;
            for (int i = et; i < G * kPC; i += 32 * kPEpiWarps) {
                const int g = i / kPC, cc = i - g * kPC;
                sbias[i] = (p.bias && d0 + cc < D) ? p.bias[g * D + d0 + cc] : 0.f;
            }
            const bool mma_ok = mbar_wait_bounded(&tfull[acc], uint32_t(st / 2) & 1u, err, p.wait_ns);
            tc_fence_after();
            epi_sync();  // the bias of this tile is in place; the last tile's gates are read

            // ---- accumulator -> bf16 gates in su (a thread holds one
            // timestep; its tensor-memory reads are issued three at a time
            // before one wait)
            {
                const int trow = 32 * lq + lane;
                const uint32_t ta = tmem + uint32_t(acc) * kAccCols + (uint32_t(32 * lq) << 16);
                constexpr int kChunks = G * kPC / 8 / 4;  // 8-column chunks per column quarter
                constexpr int kBatch = 3;
                static_assert(kChunks % kBatch == 0, "chunk batches");
#pragma unroll
                for (int k0 = 0; k0 < kChunks; k0 += kBatch) {
                    float v[kBatch][8];
#pragma unroll
                    for (int k = 0; k < kBatch; ++k) tmem_ld8(ta + uint32_t((cq * kChunks + k0 + k) * 8), v[k]);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < kBatch; ++k) {
                        const int col = (cq * kChunks + k0 + k) * 8;  // accumulator column = g * kPC + channel
                        uint32_t pk[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float x0 = mma_ok ? v[k][2 * i] + sbias[col + 2 * i] : 0.f;
                            const float x1 = mma_ok ? v[k][2 * i + 1] + sbias[col + 2 * i + 1] : 0.f;
                            pk[i] = uint32_t(bf16_bits_rn(x0)) | (uint32_t(bf16_bits_rn(x1)) << 16);
                        }
                        // lanes 2i and 2i+1 hold timesteps 2i and 2i+1: the even
                        // lane writes the pairs of channels col..col+3, the
                        // odd lane those of col+4..col+7
                        const bool odd = lane & 1;
                        const uint32_t r0 = __shfl_xor_sync(0xffffffffu, odd ? pk[0] : pk[2], 1);
                        const uint32_t r1 = __shfl_xor_sync(0xffffffffu, odd ? pk[1] : pk[3], 1);
                        uint4 q;
                        if (!odd) {
                            q = make_uint4(__byte_perm(pk[0], r0, 0x5410), __byte_perm(pk[0], r0, 0x7632),
                                           __byte_perm(pk[1], r1, 0x5410), __byte_perm(pk[1], r1, 0x7632));
                        } else {
                            q = make_uint4(__byte_perm(r0, pk[2], 0x5410), __byte_perm(r0, pk[2], 0x7632),
                                           __byte_perm(r1, pk[3], 0x5410), __byte_perm(r1, pk[3], 0x7632));
                        }
                        *reinterpret_cast<uint4*>(su + (trow >> 1) * LY::su_row + (col + (odd ? 4 : 0)) * 4) = q;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);  // this warp is done with the accumulator
            epi_sync();  // su complete


            // ---- Newton pass 0 on the tile: row group rg, channel c
            const bool cv = d0 + c < D;
            float aw[G];
#pragma unroll
            for (int g = 0; g < G; ++g) aw[g] = cv ? p.a[g * D + d0 + c] : 0.f;
            // state before step l0 at H^0
            const float hp = (l0 == 0 && p.h0 && cv) ? p.h0[b * D + d0 + c] : 0.f;
            // gate g of timesteps r, r + 1 (r even) as a pair
            auto gate2 = [&](int r, int g) {
                const uint32_t x = *reinterpret_cast<const uint32_t*>(su + (r >> 1) * LY::su_row + (g * kPC + c) * 4);
                return make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
            };
            float Jm[kRows], Ov[kRows];  // the step maps, kept for the second sweep
            float r0max = 0.f;
            Map qa = Map::identity();
            const float2 aw2[G] = {bc2(aw[0]), bc2(aw[1]), bc2(aw[2])};
            // four steps per evaluation: steps i, i+1 in the pair lanes of row
            // "a", steps i+2, i+3 in those of row "b" (they share reciprocals)
#pragma unroll
            for (int i = 0; i < kRows; i += 4) {
                float2 sa = make_float2(r0 + i == 0 ? hp : 0.f, 0.f), sb = bc2(0.f);
                float2 ua[G], ub[G], fa, fb;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    ua[g] = gate2(r0 + i, g);
                    ub[g] = gate2(r0 + i + 2, g);
                }
                Aff2<1> ja, jb;
                Cell::Packed::Rows2::eval(&sa, ua, &sb, ub, aw2, &fa, &fb, ja, jb);
                const float sv[4] = {sa.x, sa.y, sb.x, sb.y};
                const float fv[4] = {fa.x, fa.y, fb.x, fb.y}, jv[4] = {ja.m.x, ja.m.y, jb.m.x, jb.m.y};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const bool lv = l0 + r0 + i + k < L;
                    Map m{jv[k], fv[k] - jv[k] * sv[k]};
                    if (!lv) m = Map::identity();  // steps beyond L leave the state as it is
                    Jm[i + k] = m.m;
                    Ov[i + k] = m.v;
                    if (lv && cv) r0max = max_keep_nan(r0max, fabsf(fv[k]));  // F(H^0)_l = 0 - f
                    qa = compose(m, qa);
                }
            }
            qagg[(rg * kPC + c) * 2 + 0] = qa.m;
            qagg[(rg * kPC + c) * 2 + 1] = qa.v;
            epi_sync();

            // epilogue warp 0: the tile's map per channel (two a lane), the
            // decoupled look-back along the sequence, the carry.  Meanwhile
            // the other warps write u to global memory from su: a thread
            // takes 8 channels of one gate for a pair of timesteps and writes
            // 16 bytes to each; a row of one gate is 128 contiguous bytes,
            // written by 8 consecutive threads (whole lines).
            if (e != 0) {
                constexpr int kSeg = G * kPC / 8;  // 8-channel pieces of a pair of timesteps
                for (int j = et - 32; j < (kPM / 2) * kSeg; j += 32 * (kPEpiWarps - 1)) {
                    const int rp = j / kSeg, q = j - rp * kSeg;
                    const int g = q / (kPC / 8), c8 = (q - g * (kPC / 8)) * 8;
                    const uint4* src = reinterpret_cast<const uint4*>(su + rp * LY::su_row + (g * kPC + c8) * 4);
                    const uint4 w0 = src[0], w1 = src[1];
                    const uint4 ev = make_uint4(__byte_perm(w0.x, w0.y, 0x5410), __byte_perm(w0.z, w0.w, 0x5410),
                                                __byte_perm(w1.x, w1.y, 0x5410), __byte_perm(w1.z, w1.w, 0x5410));
                    const uint4 od = make_uint4(__byte_perm(w0.x, w0.y, 0x7632), __byte_perm(w0.z, w0.w, 0x7632),
                                                __byte_perm(w1.x, w1.y, 0x7632), __byte_perm(w1.z, w1.w, 0x7632));
                    const long long l = l0 + 2 * rp;
                    if (d0 + c8 < D) {
                        if (l < L) *reinterpret_cast<uint4*>(p.u + ((b * L + l) * G + g) * D + d0 + c8) = ev;
                        if (l + 1 < L) *reinterpret_cast<uint4*>(p.u + ((b * L + l + 1) * G + g) * D + d0 + c8) = od;
                    }
                }
            } else {
                const unsigned t_agg = 1u, t_incl = 2u;
                Map ta[2];
                float carry[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int cj = lane + 32 * j;
                    Map a2 = Map::identity();
#pragma unroll
                    for (int q = 0; q < kPRowGroups; ++q)
                        a2 = compose(Map{qagg[(q * kPC + cj) * 2], qagg[(q * kPC + cj) * 2 + 1]}, a2);
                    ta[j] = a2;
                    carry[j] = (l0 == 0 && p.h0 && d0 + cj < D) ? p.h0[b * D + d0 + cj] : 0.f;
                }
                unsigned long long* mine = p.desc + (size_t)t * kPDescWords;
                bool ok = true;
                if (mc > 0) {
                    st_words2(mine + lane * 4, tag_word(ta[0].m, t_agg), tag_word(ta[0].v, t_agg));
                    st_words2(mine + lane * 4 + 2, tag_word(ta[1].m, t_agg), tag_word(ta[1].v, t_agg));
                    Map ac[2] = {Map::identity(), Map::identity()};
                    int jt = t - BSf;
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
                                carry[0] = fmaf(ac[0].m, __uint_as_float(unsigned(wi0)), ac[0].v);
                                carry[1] = fmaf(ac[1].m, __uint_as_float(unsigned(wi1)), ac[1].v);
                                resolved = true;
                            } else if (unsigned(wa0 >> 32) == t_agg && unsigned(wa1 >> 32) == t_agg &&
                                       unsigned(wa2 >> 32) == t_agg && unsigned(wa3 >> 32) == t_agg) {
                                ac[0] = compose(ac[0], Map{__uint_as_float(unsigned(wa0)), __uint_as_float(unsigned(wa1))});
                                ac[1] = compose(ac[1], Map{__uint_as_float(unsigned(wa2)), __uint_as_float(unsigned(wa3))});
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
                    const float i0 = fmaf(ta[0].m, carry[0], ta[0].v), i1 = fmaf(ta[1].m, carry[1], ta[1].v);
                    st_words2(mine + kPDescAgg + lane * 2, tag_word(i0, t_incl), tag_word(i1, t_incl));
                }
                scarry[lane] = carry[0];
                scarry[lane + 32] = carry[1];
                if (lane == 0) s_flag[0] = ok ? 0 : 1;
            }
            epi_sync();

            // state entering this row group, then H^1 and the residual of H^1
            float r1max = 0.f;
            if (!s_flag[0]) {
                float y = scarry[c];
                for (int q = 0; q < rg; ++q) y = fmaf(qagg[(q * kPC + c) * 2], y, qagg[(q * kPC + c) * 2 + 1]);
                float hv[kRows + 1];  // H^1 before step r0, then at steps r0 .. r0 + kRows - 1
                hv[0] = y;
#pragma unroll
                for (int i = 0; i < kRows; ++i) hv[i + 1] = fmaf(Jm[i], hv[i], Ov[i]);
                // residual of H^1, four steps per evaluation as above
#pragma unroll
                for (int i = 0; i < kRows; i += 4) {
                    const float2 sa = make_float2(hv[i], hv[i + 1]), sb = make_float2(hv[i + 2], hv[i + 3]);
                    float2 ua[G], ub[G], fa, fb;
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        ua[g] = gate2(r0 + i, g);
                        ub[g] = gate2(r0 + i + 2, g);
                    }
                    Cell::Packed::Rows2::value(&sa, ua, &sb, ub, aw2, &fa, &fb);
                    const float fv[4] = {fa.x, fa.y, fb.x, fb.y};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const long long l = l0 + r0 + i + k;
                        if (l < L && cv) {
                            r1max = max_keep_nan(r1max, fabsf(hv[i + k + 1] - fv[k]));
                            __stcg(p.h + (b * L + l) * D + d0 + c, hv[i + k + 1]);
                        }
                    }
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                r0max = max_keep_nan(r0max, __shfl_xor_sync(0xffffffffu, r0max, off));
                r1max = max_keep_nan(r1max, __shfl_xor_sync(0xffffffffu, r1max, off));
            }
            if (lane == 0) {
                sred[e] = r0max;
                sred[kPEpiWarps + e] = r1max;
            }
            epi_sync();
            if (et == 0) {
                float x0 = 0.f, x1 = 0.f;
                for (int i = 0; i < kPEpiWarps; ++i) {
                    x0 = max_keep_nan(x0, sred[i]);
                    x1 = max_keep_nan(x1, sred[kPEpiWarps + i]);
                }
                atomicMax(&hdr->res0, __float_as_uint(x0) & 0x7fffffffu);
                atomicMax(&hdr->res[0], __float_as_uint(x1) & 0x7fffffffu);
            }
            if (s_flag[0]) break;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tmem, 2 * kAccCols);
    if (tid == 0 && blockIdx.x == 0) hdr->k0 = 1;  // the fused solve continues with pass 1
}

}  // namespace pararnn
