// C ABI of libpararnn.so: argument checks, workspace layout, TMA descriptors
// and kernel launches for the ParaRNN Newton solves, adjoints and baselines.
// The entry points and their conventions are documented in include/pararnn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "pararnn.h"
#include "pararnn_internal.h"
#include "device_common.cuh"
#include "cells.cuh"
#include "newton.cuh"
#include "newton_ws.cuh"
#include "sequential.cuh"
#include "decode.cuh"
#include "segment.cuh"
#include "adjoint.cuh"
#include "da_reduce.cuh"
#include "selftest.cuh"
#include "adjoint_ws.cuh"
#include "linear_scan.cuh"
#include "project.cuh"

using namespace pararnn;

namespace {

thread_local char t_err[512] = "";
std::atomic<unsigned long long> g_launches{0};

pararnn_status fail(pararnn_status s, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_err, sizeof(t_err), fmt, ap);
    va_end(ap);
    return s;
}

#define CUDA_TRY(expr)                                                                        \
    do {                                                                                      \
        cudaError_t e_ = (expr);                                                              \
        if (e_ != cudaSuccess)                                                                \
            return fail(PARARNN_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_));    \
    } while (0)

#define TRY(expr)                                 \
    do {                                          \
        pararnn_status s_ = (expr);               \
        if (s_ != PARARNN_OK) return s_;          \
    } while (0)

constexpr size_t kSelftestWorkspace = 16384;
#ifndef PARARNN_WS_GRU_WARPS
#define PARARNN_WS_GRU_WARPS 15
#endif
#ifndef PARARNN_WS_LSTM_WARPS
#define PARARNN_WS_LSTM_WARPS 7
#endif
// row pairs per tile (two steps each); fp32 gates need twice the staging
// space, so their tiles are half as long
template <class UT> constexpr int gru_tile_arg() { return sizeof(UT) == 2 ? PARARNN_WS_GRU_WARPS : PARARNN_WS_GRU_WARPS / 2; }
template <class UT> constexpr int lstm_tile_arg() { return sizeof(UT) == 2 ? PARARNN_WS_LSTM_WARPS : PARARNN_WS_LSTM_WARPS / 2; }
template <class UT> constexpr int gru_lc() { return 2 * gru_tile_arg<UT>(); }
template <class UT> constexpr int lstm_lc() { return 2 * lstm_tile_arg<UT>(); }
// workspace sizing uses the shortest tile (most tiles) of either input dtype
constexpr int kLcGru = gru_lc<float>() < gru_lc<uint16_t>() ? gru_lc<float>() : gru_lc<uint16_t>();
constexpr int kLcLstm = lstm_lc<float>() < lstm_lc<uint16_t>() ? lstm_lc<float>() : lstm_lc<uint16_t>();

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Shape {
    long long B, L, D;
    int S, n_chunks, n_tiles, Lc;
};

bool shape_ok(long long B, long long L, long long D) { return B >= 1 && L >= 1 && D >= 1; }

pararnn_status make_shape(long long B, long long L, long long D, int Lc, Shape* s)
{
    if (!shape_ok(B, L, D)) return fail(PARARNN_ERR_INVALID_ARG, "B, L, D must be >= 1 (got %lld, %lld, %lld)", B, L, D);
    if (D % 8 != 0) return fail(PARARNN_ERR_UNSUPPORTED, "D must be a multiple of 8 (got %lld)", D);
    if (L > INT_MAX / 2 || B > INT_MAX / 2 || D > INT_MAX / 2)
        return fail(PARARNN_ERR_INVALID_ARG, "dimension too large");
    if ((double)B * (double)L * (double)D * 16.0 >= 1099511627776.0)
        return fail(PARARNN_ERR_INVALID_ARG, "B*L*D too large (gate strides must stay below 2^40 bytes)");
    s->B = B;
    s->L = L;
    s->D = D;
    s->Lc = Lc;
    s->S = int((D + kDc - 1) / kDc);
    s->n_chunks = int((L + Lc - 1) / Lc);
    const long long nt = (long long)s->n_chunks * B * s->S;
    if (nt > INT_MAX / 4) return fail(PARARNN_ERR_INVALID_ARG, "too many tiles");
    s->n_tiles = int(nt);
    return PARARNN_OK;
}

struct ScanLayout {
    size_t desc, extra, total;
};

// header | look-back descriptors (tagged 64-bit words; one per tile, or
// n_desc of them) | extra (boundary / partial sums).  Header and descriptors
// are zeroed before every launch.
ScanLayout scan_layout(const Shape& s, int desc_words, size_t extra_bytes, long long n_desc = -1)
{
    ScanLayout ly;
    ly.desc = sizeof(WsHeader);
    ly.extra = align256(ly.desc + size_t(n_desc < 0 ? s.n_tiles : n_desc) * desc_words * 8);
    ly.total = align256(ly.extra + extra_bytes);
    return ly;
}

// the fused solve keeps one look-back descriptor per group of chunks
long long solve_descs(const Shape& s) { return solve_desc_count(s.n_chunks, s.B * s.S); }

// Whether the solve's look-backs step back over predecessors' aggregates.
// Every CTA holds about two groups, so grid / sequences groups of one
// sequence are in flight.  With few of them (many sequences) a group's
// predecessor publishes its inclusive value about as soon as a step back
// would find anything, and waiting for it -- with no aggregates published or
// read at all -- is faster (measured: ParaLSTM B=8 L=4096 D=1024 1.32 ms
// against 1.97 ms stepping back; ParaGRU 0.620 against 0.646 ms); with many
// (one sequence of 2048 channels: 16 slabs over 148 CTAs) a chain of
// inclusive values paces the pass and stepping back is faster (ParaGRU B=1
// L=65536 D=2048: 2.81 against 3.17 ms).
int solve_lookback_walks(int grid, long long sequences) { return grid >= 4 * sequences ? 1 : 0; }

// Whether ParaGRU passes that continue may leave residuals out once a tile has
// found one above tol.  It pays where each CTA runs several tiles a pass; with
// about one or two (short sequences) the flag arrives too late to spare much
// and its checks cost more than they save (measured at B1 D2048: L = 512
// 0.0615 ms without, 0.065 with; L = 2048 0.137 with, 0.141 without).
int solve_skips_residuals(long long n_tiles, int grid) { return n_tiles >= 4LL * grid ? 1 : 0; }

size_t solve_bnd_bytes(const Shape& s, int NS)
{
    return size_t(2) * NS * s.B * s.n_chunks * s.S * kDc * 4;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pararnn_status check_ptr(const void* p, const char* name, bool required)
{
    if (!p) return required ? fail(PARARNN_ERR_INVALID_ARG, "%s is NULL", name) : PARARNN_OK;
    if (!aligned16(p)) return fail(PARARNN_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return PARARNN_OK;
}

pararnn_status check_dtype(pararnn_dtype dt)
{
    if (dt != PARARNN_F32 && dt != PARARNN_BF16) return fail(PARARNN_ERR_INVALID_ARG, "unknown u dtype %d", int(dt));
    return PARARNN_OK;
}

pararnn_status check_workspace(const void* ws, size_t bytes, size_t need)
{
    if (!ws) return fail(PARARNN_ERR_WORKSPACE, "workspace is NULL");
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(PARARNN_ERR_WORKSPACE, "workspace is not 256-byte aligned");
    if (bytes < need) return fail(PARARNN_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", bytes, need);
    return PARARNN_OK;
}

// ---------------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Gate tensor [B][L][G][D] -> box [1][rows][G][kDc] (or a single gate g_box = 1).
pararnn_status map_gates(CUtensorMap* m, const void* u, pararnn_dtype dt, int G, int g_box, const Shape& s,
                         int rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(PARARNN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    const cuuint64_t es = dt == PARARNN_BF16 ? 2 : 4;
    cuuint64_t dims[4] = {cuuint64_t(s.D), cuuint64_t(G), cuuint64_t(s.L), cuuint64_t(s.B)};
    cuuint64_t strides[3] = {cuuint64_t(s.D) * es, cuuint64_t(G) * s.D * es, cuuint64_t(s.L) * G * s.D * es};
    cuuint32_t box[4] = {cuuint32_t(kDc), cuuint32_t(g_box), cuuint32_t(rows), 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    CUresult r = enc(m, dt == PARARNN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                     const_cast<void*>(u), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PARARNN_ERR_CUDA, "cuTensorMapEncodeTiled(gates) failed: %d", int(r));
    return PARARNN_OK;
}

// State tensor [B][L][D] fp32 -> box [1][rows][kDc].
pararnn_status map_state(CUtensorMap* m, const float* x, const Shape& s, int rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(PARARNN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {cuuint64_t(s.D), cuuint64_t(s.L), cuuint64_t(s.B)};
    cuuint64_t strides[2] = {cuuint64_t(s.D) * 4, cuuint64_t(s.L) * s.D * 4};
    cuuint32_t box[3] = {cuuint32_t(kDc), cuuint32_t(rows), 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(x), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PARARNN_ERR_CUDA, "cuTensorMapEncodeTiled(state) failed: %d", int(r));
    return PARARNN_OK;
}

// Recurrence weights a [G][D] fp32: box = one slab of kDc channels, all gates.
pararnn_status map_weights(CUtensorMap* m, const float* a, int G, const Shape& s)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(PARARNN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {cuuint64_t(s.D), cuuint64_t(G)};
    cuuint64_t strides[1] = {cuuint64_t(s.D) * 4};
    cuuint32_t box[2] = {cuuint32_t(kDc), cuuint32_t(G)};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(a), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PARARNN_ERR_CUDA, "cuTensorMapEncodeTiled(weights) failed: %d", int(r));
    return PARARNN_OK;
}

// Chunk boundary rows [2][NS][B][n_chunks][S*kDc] fp32, seen as 3-D
// {D channels, n_chunks, 2*NS*B rows}: box = one slab of one row.
pararnn_status map_bnd(CUtensorMap* m, const float* bnd, int NS, const Shape& s)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(PARARNN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    const cuuint64_t row = cuuint64_t(s.S) * kDc * 4;
    cuuint64_t dims[3] = {cuuint64_t(s.D), cuuint64_t(s.n_chunks), cuuint64_t(2) * NS * s.B};
    cuuint64_t strides[2] = {row, row * cuuint64_t(s.n_chunks)};
    cuuint32_t box[3] = {cuuint32_t(kDc), 1u, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(bnd), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PARARNN_ERR_CUDA, "cuTensorMapEncodeTiled(boundary) failed: %d", int(r));
    return PARARNN_OK;
}

pararnn_status device_info(int* sms)
{
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    CUDA_TRY(cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev));
    int coop = 0;
    CUDA_TRY(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev));
    if (!coop) return fail(PARARNN_ERR_UNSUPPORTED, "device does not support cooperative launch");
    return PARARNN_OK;
}

template <class K>
pararnn_status resident_grid(K kern, size_t smem, int n_tiles, int* grid, int threads)
{
    int sms = 0;
    TRY(device_info(&sms));
    CUDA_TRY(cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  int(smem)));
    int occ = 0;
    CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem));
    if (occ < 1) return fail(PARARNN_ERR_CUDA, "kernel does not fit on an SM (smem %zu)", smem);
    *grid = std::max(1, std::min(n_tiles, occ * sms));
    return PARARNN_OK;
}

// ----------------------------------------------------------------- solves

// in: where the first pass reads the states (segment passes: the given
// iterate; NULL = st); slin, warm: see NewtonParams.
template <class Cell, class UT, int T, bool Seg, int LB>
pararnn_status launch_newton_k(const Shape& s, const void* u, pararnn_dtype dt, const float* a,
                               const float* const s0[2], float* const st[2], float tol, int max_iters, void* ws,
                               cudaStream_t stream, const float* const* in, const float* const* slin, int warm,
                               bool zero_ws)
{
    constexpr int NS = Cell::NS;
    constexpr int desc_words = TileDesc<typename Cell::Map, NS>::words;
    using KL = NewtonWsLayout<Cell, UT, T>;  // T = compute warps (two steps each)
    auto kern = newton_solve_ws_kernel<Cell, UT, T, Seg, LB>;
    constexpr int threads = KL::threads;
    // the TMA boxes must be exactly the kernel's tile
    if (s.Lc != KL::Lc) return fail(PARARNN_ERR_INVALID_ARG, "internal: tile rows %d != kernel rows %d", s.Lc, KL::Lc);
    const ScanLayout ly = scan_layout(s, desc_words, solve_bnd_bytes(s, NS), solve_descs(s));
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    // header + descriptors; waiting look-backs (LB = 0) use the leading part
    // of the region only, as descriptors without aggregates
    const size_t zero_bytes =
        LB == 0 ? ly.desc + size_t(solve_descs(s)) * TileDesc<typename Cell::Map, NS, false>::words * 8 : ly.extra;
    if (zero_ws) CUDA_TRY(cudaMemsetAsync(ws, 0, zero_bytes, stream));

    CUtensorMap tu, t0, t1;
    TRY(map_gates(&tu, u, dt, Cell::G, Cell::G, s, KL::Lc));
    const float* src[2] = {in ? in[0] : st[0], in ? in[NS - 1] : st[NS - 1]};
    TRY(map_state(&t0, src[0], s, KL::Lc));
    TRY(map_state(&t1, src[1], s, KL::Lc));

    NewtonParams p;
    p.a = a;
    p.s0[0] = s0[0];
    p.s0[1] = s0[1];
    p.st[0] = st[0];
    p.st[1] = st[1];
    p.B = s.B;
    p.L = s.L;
    p.D = s.D;
    p.S = s.S;
    p.n_chunks = s.n_chunks;
    p.n_tiles = s.n_tiles;
    p.tol = tol;
    p.max_iters = max_iters;
    p.hdr = reinterpret_cast<WsHeader*>(wsb);
    p.desc = reinterpret_cast<unsigned long long*>(wsb + ly.desc);
    p.bnd = reinterpret_cast<float*>(wsb + ly.extra);
    p.wait_ns = kWaitLimitNs;
    if (Seg) {  // into the zeroed header (pageable source: consumed before the call returns)
        struct {
            unsigned long long lin[2];
            int warm;
        } seg = {{slin ? reinterpret_cast<unsigned long long>(slin[0]) : 0ull,
                  slin ? reinterpret_cast<unsigned long long>(slin[1]) : 0ull},
                 warm};
        static_assert(offsetof(WsHeader, seg_warm) == offsetof(WsHeader, seg_lin) + 16, "header layout");
        CUDA_TRY(cudaMemcpyAsync(wsb + offsetof(WsHeader, seg_lin), &seg, 20, cudaMemcpyHostToDevice, stream));
    }
    if (warm && s.n_chunks > 1) {
        const long long n = (long long)NS * s.B * (s.n_chunks - 1) * (s.D / 4);
        bnd_gather_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(src[0], src[1], p.bnd, NS, s.B, s.L, s.D,
                                                                          s.n_chunks, KL::Lc, s.S * kDc);
        CUDA_TRY(cudaGetLastError());
        g_launches.fetch_add(1, std::memory_order_relaxed);
    }

    int grid = 0;
    TRY(resident_grid(kern, KL::smem_bytes, s.n_tiles, &grid, threads));
    p.lb_walk = LB;
    p.skip_res = solve_skips_residuals(s.n_tiles, grid);
    CUtensorMap ta, tb;
    TRY(map_weights(&ta, a, Cell::G, s));
    TRY(map_bnd(&tb, p.bnd, NS, s));
    void* args[] = {(void*)&tu, (void*)&t0, (void*)&t1, (void*)&ta, (void*)&tb, (void*)&p};
    CUDA_TRY(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(threads), args,
                                         KL::smem_bytes, stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PARARNN_OK;
}

// The fused solve in the look-back mode that suits the shape (see
// solve_lookback_walks): stepping back over aggregates, or waiting for
// inclusive values.  Both kernel variants run one CTA per SM.
template <class Cell, class UT, int T, bool Seg = false>
pararnn_status launch_newton(const Shape& s, const void* u, pararnn_dtype dt, const float* a, const float* const s0[2],
                             float* const st[2], float tol, int max_iters, void* ws, cudaStream_t stream,
                             const float* const* in = nullptr, const float* const* slin = nullptr, int warm = 0,
                             bool zero_ws = true)
{
    int sms = 0;
    TRY(device_info(&sms));
    if (solve_lookback_walks(std::min(s.n_tiles, sms), s.B * s.S))
        return launch_newton_k<Cell, UT, T, Seg, 1>(s, u, dt, a, s0, st, tol, max_iters, ws, stream, in, slin, warm,
                                                    zero_ws);
    return launch_newton_k<Cell, UT, T, Seg, 0>(s, u, dt, a, s0, st, tol, max_iters, ws, stream, in, slin, warm,
                                                zero_ws);
}

size_t solve_ws_bytes(int cell, long long B, long long L, long long D)
{
    if (!shape_ok(B, L, D) || D % 8 != 0) return 0;
    Shape s;
    char saved[sizeof(t_err)];
    memcpy(saved, t_err, sizeof(t_err));
    pararnn_status st = make_shape(B, L, D, cell == 0 ? kLcGru : kLcLstm, &s);
    memcpy(t_err, saved, sizeof(t_err));
    if (st != PARARNN_OK) return 0;
    if (cell == 0) return scan_layout(s, TileDesc<Aff<1>, 1>::words, solve_bnd_bytes(s, 1), solve_descs(s)).total;
    return scan_layout(s, TileDesc<Aff<2>, 2>::words, solve_bnd_bytes(s, 2), solve_descs(s)).total;
}

// Host-side argument checks of a solve (everything but the workspace); no
// device call.
pararnn_status solve_args(int cell, const void* u, pararnn_dtype dt, const float* a, const float* c0, const float* h0,
                          const float* c, const float* h, long long B, long long L, long long D, float tol,
                          int max_iters)
{
    TRY(check_dtype(dt));
    TRY(check_ptr(u, "u", true));
    TRY(check_ptr(a, "a", true));
    TRY(check_ptr(h0, "h0", false));
    TRY(check_ptr(h, "h", true));
    if (cell == 1) {
        TRY(check_ptr(c0, "c0", false));
        TRY(check_ptr(c, "c", true));
    }
    if (!(tol >= 0.0f) || !std::isfinite(tol)) return fail(PARARNN_ERR_INVALID_ARG, "tol must be finite and >= 0");
    if (max_iters < 0) return fail(PARARNN_ERR_INVALID_ARG, "max_iters must be >= 0");
    Shape s;
    return make_shape(B, L, D, cell == 0 ? kLcGru : kLcLstm, &s);
}

pararnn_status solve_async(int cell, const void* u, pararnn_dtype dt, const float* a, const float* c0, const float* h0,
                           float* c, float* h, long long B, long long L, long long D, float tol, int max_iters,
                           void* ws, size_t ws_bytes, cudaStream_t stream)
{
    t_err[0] = '\0';
    TRY(solve_args(cell, u, dt, a, c0, h0, c, h, B, L, D, tol, max_iters));
    Shape s;
    TRY(check_workspace(ws, ws_bytes, solve_ws_bytes(cell, B, L, D)));
    if (cell == 0) {
        const float* s0[2] = {h0, nullptr};
        float* st[2] = {h, nullptr};
        if (dt == PARARNN_BF16) {
            TRY(make_shape(B, L, D, gru_lc<uint16_t>(), &s));
            return launch_newton<GruCell, uint16_t, gru_tile_arg<uint16_t>()>(s, u, dt, a, s0, st, tol, max_iters, ws, stream);
        }
        TRY(make_shape(B, L, D, gru_lc<float>(), &s));
        return launch_newton<GruCell, float, gru_tile_arg<float>()>(s, u, dt, a, s0, st, tol, max_iters, ws, stream);
    }
    const float* s0[2] = {c0, h0};
    float* st[2] = {c, h};
    if (dt == PARARNN_BF16) {
        TRY(make_shape(B, L, D, lstm_lc<uint16_t>(), &s));
        return launch_newton<LstmCell, uint16_t, lstm_tile_arg<uint16_t>()>(s, u, dt, a, s0, st, tol, max_iters, ws, stream);
    }
    TRY(make_shape(B, L, D, lstm_lc<float>(), &s));
    return launch_newton<LstmCell, float, lstm_tile_arg<float>()>(s, u, dt, a, s0, st, tol, max_iters, ws, stream);
}

// ------------------------------------------------ segments of a sequence

// One Newton pass over a segment (see segment.cuh): from s_in (NULL: the zero
// guess), linearising the segment's first step at s_lin, with s_carry as the
// state entering it; the segment's last-step states are copied to s_end.
// Components are stacked: s_in, s_out [NS][B][Ls][D]; s_lin, s_carry, s_end [NS][B][D].
pararnn_status segment_pass_async(int cell, const void* u, pararnn_dtype dt, const float* a, const float* s_in,
                                  const float* s_lin, const float* s_carry, float* s_out, float* s_end, long long B,
                                  long long L, long long D, void* ws, size_t ws_bytes, cudaStream_t stream)
{
    t_err[0] = '\0';
    TRY(check_dtype(dt));
    TRY(check_ptr(u, "u", true));
    TRY(check_ptr(a, "a", true));
    TRY(check_ptr(s_in, "s_in", false));
    TRY(check_ptr(s_lin, "s_lin", false));
    TRY(check_ptr(s_carry, "s_carry", false));
    TRY(check_ptr(s_out, "s_out", true));
    TRY(check_ptr(s_end, "s_end", false));
    Shape s;
    TRY(make_shape(B, L, D, cell == 0 ? kLcGru : kLcLstm, &s));
    TRY(check_workspace(ws, ws_bytes, solve_ws_bytes(cell, B, L, D)));
    const int NS = cell == 0 ? 1 : 2;
    const long long per = B * L * D, per0 = B * D;
    if (s_in && s_in != s_out) {
        // in place is fine (a tile reads only its own rows, and the states
        // entering its chunk come from the boundary rows); a shifted overlap
        // would let one tile overwrite rows another still reads
        const uintptr_t i0 = reinterpret_cast<uintptr_t>(s_in), o0 = reinterpret_cast<uintptr_t>(s_out);
        const uintptr_t len = uintptr_t(NS * per) * 4;
        if (i0 < o0 + len && o0 < i0 + len)
            return fail(PARARNN_ERR_INVALID_ARG, "s_out overlaps s_in without being s_in itself");
    }
    const float* s0[2] = {s_carry, s_carry && NS == 2 ? s_carry + per0 : nullptr};
    float* st[2] = {s_out, NS == 2 ? s_out + per : nullptr};
    const float* in[2] = {s_in ? s_in : s_out, s_in ? s_in + (NS - 1) * per : s_out + (NS - 1) * per};
    const float* lin[2] = {s_lin, s_lin && NS == 2 ? s_lin + per0 : nullptr};
    // no device-side decision: exactly one pass (tol < 0 is never met)
    const float tol = -1.0f;
    const int warm = s_in ? 1 : 0;
    pararnn_status r;
    if (cell == 0) {
        if (dt == PARARNN_BF16) {
            TRY(make_shape(B, L, D, gru_lc<uint16_t>(), &s));
            r = launch_newton<GruCell, uint16_t, gru_tile_arg<uint16_t>(), true>(s, u, dt, a, s0, st, tol, 1, ws,
                                                                                stream, in, lin, warm);
        } else {
            TRY(make_shape(B, L, D, gru_lc<float>(), &s));
            r = launch_newton<GruCell, float, gru_tile_arg<float>(), true>(s, u, dt, a, s0, st, tol, 1, ws, stream, in,
                                                                          lin, warm);
        }
    } else {
        if (dt == PARARNN_BF16) {
            TRY(make_shape(B, L, D, lstm_lc<uint16_t>(), &s));
            r = launch_newton<LstmCell, uint16_t, lstm_tile_arg<uint16_t>(), true>(s, u, dt, a, s0, st, tol, 1, ws,
                                                                                  stream, in, lin, warm);
        } else {
            TRY(make_shape(B, L, D, lstm_lc<float>(), &s));
            r = launch_newton<LstmCell, float, lstm_tile_arg<float>(), true>(s, u, dt, a, s0, st, tol, 1, ws, stream,
                                                                            in, lin, warm);
        }
    }
    TRY(r);
    if (s_end) {
        for (int q = 0; q < NS; ++q)
            CUDA_TRY(cudaMemcpy2DAsync(s_end + q * per0, size_t(D) * 4, st[q] + (L - 1) * D, size_t(L) * D * 4,
                                       size_t(D) * 4, size_t(B), cudaMemcpyDeviceToDevice, stream));
    }
    return PARARNN_OK;
}

long long segment_record_floats(int cell, long long BD)
{
    return cell == 0 ? SegRecord<GruCell>::floats(BD) : SegRecord<LstmCell>::floats(BD);
}

// fold parts [nf][NC][B][D] of segment_fold_kernel
size_t segment_fold_ws_bytes(int cell, long long B, long long L, long long D)
{
    if (!shape_ok(B, L, D) || D % 8 != 0) return 0;
    const long long steps = fold_steps(L), nf = (L - 1 + steps - 1) / steps;
    return align256(size_t(std::max(nf, 1ll)) * (cell == 0 ? 2 : 6) * B * D * 4);
}

template <class Cell, class UT>
pararnn_status launch_fold(const UT* u, const float* a, const float* s_in, float* rec, float* part, long long B,
                           long long L, long long D, cudaStream_t stream)
{
    using R = SegRecord<Cell>;
    const long long BD = B * D;
    unsigned* res = reinterpret_cast<unsigned*>(rec + R::F * BD);
    CUDA_TRY(cudaMemsetAsync(res, 0, 16, stream));
    const long long steps = fold_steps(L);
    const int nf = int((L - 1 + steps - 1) / steps);
    if (nf > 0) {
        const long long threads = B * (D / 4);
        const dim3 grid(unsigned((threads + 127) / 128), unsigned(nf)), block(128);
        segment_fold_kernel<Cell, UT><<<grid, block, 0, stream>>>(u, a, s_in, part, res, B, L, D, int(steps));
        CUDA_TRY(cudaGetLastError());
        g_launches.fetch_add(1, std::memory_order_relaxed);
    }
    segment_record_kernel<Cell, UT><<<unsigned((BD + 255) / 256), 256, 0, stream>>>(u, s_in, part, nf, rec, B, L, D);
    CUDA_TRY(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PARARNN_OK;
}

// A segment's record for the iteration from H^k = s_in [NS][B][Ls][D] (NULL:
// the zero guess): see SegRecord in segment.cuh.
pararnn_status segment_fold_async(int cell, const void* u, pararnn_dtype dt, const float* a, const float* s_in,
                                  float* rec, long long B, long long L, long long D, void* ws, size_t ws_bytes,
                                  cudaStream_t stream)
{
    t_err[0] = '\0';
    TRY(check_dtype(dt));
    TRY(check_ptr(u, "u", true));
    TRY(check_ptr(a, "a", true));
    TRY(check_ptr(s_in, "s_in", false));
    TRY(check_ptr(rec, "record", true));
    Shape s;
    TRY(make_shape(B, L, D, 1, &s));
    TRY(check_workspace(ws, ws_bytes, segment_fold_ws_bytes(cell, B, L, D)));
    float* part = static_cast<float*>(ws);
    if (cell == 0) {
        if (dt == PARARNN_BF16)
            return launch_fold<GruCell, uint16_t>(static_cast<const uint16_t*>(u), a, s_in, rec, part, B, L, D, stream);
        return launch_fold<GruCell, float>(static_cast<const float*>(u), a, s_in, rec, part, B, L, D, stream);
    }
    if (dt == PARARNN_BF16)
        return launch_fold<LstmCell, uint16_t>(static_cast<const uint16_t*>(u), a, s_in, rec, part, B, L, D, stream);
    return launch_fold<LstmCell, float>(static_cast<const float*>(u), a, s_in, rec, part, B, L, D, stream);
}

// Every segment's record (R of them, in segment order) -> the state entering
// segment `index` and the state its first step is linearised at, and the
// residual of the iterate over all segments.
pararnn_status segment_combine_async(int cell, const float* recs, int n_seg, int index, const float* a,
                                     const float* s0, float* carry, float* lin, float* residual, long long B,
                                     long long D, cudaStream_t stream)
{
    t_err[0] = '\0';
    TRY(check_ptr(recs, "records", true));
    TRY(check_ptr(a, "a", true));
    TRY(check_ptr(s0, "s0", false));
    TRY(check_ptr(carry, "carry", true));
    TRY(check_ptr(lin, "lin", true));
    if (!residual) return fail(PARARNN_ERR_INVALID_ARG, "residual is NULL");
    if (n_seg < 1) return fail(PARARNN_ERR_INVALID_ARG, "n_segments must be >= 1 (got %d)", n_seg);
    if (index < 0 || index >= n_seg)
        return fail(PARARNN_ERR_INVALID_ARG, "index %d is not a segment of %d", index, n_seg);
    if (B < 1 || D < 1 || D % 8 != 0) return fail(B < 1 || D < 1 ? PARARNN_ERR_INVALID_ARG : PARARNN_ERR_UNSUPPORTED,
                                                  "B, D must be >= 1 and D a multiple of 8");
    const long long BD = B * D;
    unsigned* res = reinterpret_cast<unsigned*>(residual);
    CUDA_TRY(cudaMemsetAsync(res, 0, 4, stream));
    const dim3 grid(unsigned((BD + 255) / 256)), block(256);
    if (cell == 0)
        segment_combine_kernel<GruCell><<<grid, block, 0, stream>>>(recs, n_seg, index, s0, a, carry, lin, res, B, D);
    else
        segment_combine_kernel<LstmCell><<<grid, block, 0, stream>>>(recs, n_seg, index, s0, a, carry, lin, res, B, D);
    CUDA_TRY(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PARARNN_OK;
}

pararnn_status read_header(const void* ws, cudaStream_t stream, WsHeader* h)
{
    if (!ws) return fail(PARARNN_ERR_WORKSPACE, "workspace is NULL");
    CUDA_TRY(cudaMemcpyAsync(h, ws, sizeof(WsHeader), cudaMemcpyDeviceToHost, stream));
    CUDA_TRY(cudaStreamSynchronize(stream));
    return PARARNN_OK;
}

pararnn_status finish_sync(void* ws, cudaStream_t stream, int* iters_out, float* residual_out)
{
    pararnn_result r;
    pararnn_status st = pararnn_read_result(ws, stream, &r);
    if (st < 0 && st != PARARNN_ERR_NONFINITE) return st;
    if (iters_out) *iters_out = r.iters;
    if (residual_out) *residual_out = r.residual;
    return st;
}

// ------------------------------------- input projection fused with pass 0

// bf16 [n2][n1][n0] (n0 contiguous) -> box {64, rows, 1} with the 128-byte
// swizzle the tensor-core operand descriptors expect.
pararnn_status map_bf16_sw128(CUtensorMap* m, const void* p, cuuint64_t n0, cuuint64_t n1, cuuint64_t n2,
                              cuuint32_t rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(PARARNN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {n0, n1, n2};
    cuuint64_t strides[2] = {n0 * 2, n0 * n1 * 2};
    cuuint32_t box[3] = {cuuint32_t(kPK), rows, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PARARNN_ERR_CUDA, "cuTensorMapEncodeTiled(projection operand) failed: %d", int(r));
    return PARARNN_OK;
}

long long project_tiles(long long B, long long L, long long D)
{
    return ((L + kPM - 1) / kPM) * B * ((D + kPC - 1) / kPC);
}

// the solve's workspace, then the fused kernel's look-back descriptors
size_t project_ws_bytes(long long B, long long L, long long D, long long Din)
{
    if (!shape_ok(B, L, D) || D % 8 != 0 || Din < 8 || Din % 8 != 0) return 0;
    const size_t solve = solve_ws_bytes(0, B, L, D);
    if (!solve) return 0;
    return align256(solve + size_t(project_tiles(B, L, D)) * kPDescWords * 8);
}

pararnn_status project_solve_async(const void* x, const void* w, const float* bias, const float* a, const float* h0,
                                   uint16_t* u, float* h, long long B, long long L, long long Din, long long D,
                                   float tol, int max_iters, void* ws, size_t ws_bytes, cudaStream_t stream)
{
    t_err[0] = '\0';
    TRY(check_ptr(x, "x", true));
    TRY(check_ptr(w, "w", true));
    TRY(check_ptr(bias, "bias", false));
    TRY(check_ptr(u, "u", true));
    TRY(solve_args(0, u, PARARNN_BF16, a, nullptr, h0, nullptr, h, B, L, D, tol, max_iters));
    if (Din < 8 || Din % 8 != 0) return fail(PARARNN_ERR_UNSUPPORTED, "Din must be a positive multiple of 8 (got %lld)", Din);
    if ((double)B * (double)L * (double)Din * 2.0 >= 1099511627776.0) return fail(PARARNN_ERR_INVALID_ARG, "x too large");
    if (project_tiles(B, L, D) > INT_MAX / 2) return fail(PARARNN_ERR_INVALID_ARG, "too many tiles");
    TRY(check_workspace(ws, ws_bytes, project_ws_bytes(B, L, D, Din)));
    Shape s;
    TRY(make_shape(B, L, D, gru_lc<uint16_t>(), &s));
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    const size_t solve = solve_ws_bytes(0, B, L, D);
    const long long nt = project_tiles(B, L, D);
    const ScanLayout ly = scan_layout(s, TileDesc<Aff<1>, 1>::words, solve_bnd_bytes(s, 1), solve_descs(s));
    CUDA_TRY(cudaMemsetAsync(ws, 0, ly.extra, stream));  // header + the solve's descriptors
    CUDA_TRY(cudaMemsetAsync(wsb + solve, 0, size_t(nt) * kPDescWords * 8, stream));

    CUtensorMap tx, tw;
    TRY(map_bf16_sw128(&tx, x, cuuint64_t(Din), cuuint64_t(L), cuuint64_t(B), kPM));
    TRY(map_bf16_sw128(&tw, w, cuuint64_t(Din), cuuint64_t(D), 3, kPC));
    ProjectParams p;
    p.bias = bias;
    p.a = a;
    p.h0 = h0;
    p.u = u;
    p.h = h;
    p.B = B;
    p.L = L;
    p.D = D;
    p.Din = Din;
    p.Sf = int((D + kPC - 1) / kPC);
    p.n_chunks = int((L + kPM - 1) / kPM);
    p.n_tiles = int(nt);
    p.hdr = reinterpret_cast<WsHeader*>(wsb);
    p.desc = reinterpret_cast<unsigned long long*>(wsb + solve);
    p.wait_ns = kWaitLimitNs;
    using PL = ProjectLayout<3>;
    int grid = 0;
    TRY(resident_grid(project_pass0_kernel, PL::smem_bytes, int(nt), &grid, kPThreads));
    void* args[] = {(void*)&tx, (void*)&tw, (void*)&p};
    CUDA_TRY(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(project_pass0_kernel), dim3(grid),
                                         dim3(kPThreads), args, PL::smem_bytes, stream));
    g_launches.fetch_add(1, std::memory_order_relaxed);

    // H^1 at the solve's chunk ends into the boundary rows pass 1 reads
    // (ring slot 1), then the fused solve from pass 1 on the same header
    float* bnd = reinterpret_cast<float*>(wsb + ly.extra);
    if (s.n_chunks > 1) {
        const long long n = (long long)s.B * (s.n_chunks - 1) * (s.D / 4);
        bnd_gather_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(h, h, bnd + size_t(s.B) * s.n_chunks * s.S * kDc,
                                                                          1, s.B, s.L, s.D, s.n_chunks, s.Lc,
                                                                          s.S * kDc);
        CUDA_TRY(cudaGetLastError());
        g_launches.fetch_add(1, std::memory_order_relaxed);
    }
    const float* s0[2] = {h0, nullptr};
    float* st[2] = {h, nullptr};
    return launch_newton<GruCell, uint16_t, gru_tile_arg<uint16_t>()>(s, u, PARARNN_BF16, a, s0, st, tol, max_iters,
                                                                      ws, stream, nullptr, nullptr, 0, false);
}

// --------------------------------------------------------------- adjoints

// Compute warps (two steps each) of the warp-specialised adjoint per cell,
// gate dtype and staged upstream components (NG; a ParaLSTM loss on h alone
// stages one, which leaves shared memory for a ninth warp); fp32 gates need
// twice the staging space, so their tiles are half as long.
#ifndef PARARNN_ADJ_GRU_WARPS
#define PARARNN_ADJ_GRU_WARPS 15
#endif
#ifndef PARARNN_ADJ_LSTM_WARPS
#define PARARNN_ADJ_LSTM_WARPS 8
#endif
#ifndef PARARNN_ADJ_LSTM_H_WARPS
#define PARARNN_ADJ_LSTM_H_WARPS 9
#endif
template <class Cell, class UT, int NG> constexpr int adj_warps()
{
    return (Cell::NS == 1 ? PARARNN_ADJ_GRU_WARPS : NG == 1 ? PARARNN_ADJ_LSTM_H_WARPS : PARARNN_ADJ_LSTM_WARPS) /
           (sizeof(UT) == 2 ? 1 : 2);
}
// workspace sizing uses the shortest tile (most tiles) of any variant
template <class Cell> constexpr int adj_lc_min()
{
    constexpr int a = adj_warps<Cell, float, Cell::NS>(), b = adj_warps<Cell, float, 1>();
    return 2 * (a < b ? a : b);
}

// Row slabs of the da reduction: about 1024 blocks of da_slab_kernel, and no
// more slabs than rows.  A function of the shape alone, so that the sums are
// added in the same order on every run.
int da_slabs(long long rows, int S, int G)
{
    const long long SG = (long long)S * G;
    return int(std::max(1LL, std::min(rows, (1024 + SG - 1) / SG)));
}

// Workspace bytes after the descriptors: the per-tile partial sums
// [B*n_chunks][S][G][kDc], then the slab sums [slabs][S][G][kDc].
size_t da_bytes(const Shape& s, int G)
{
    const long long rows = s.B * s.n_chunks;
    return (size_t(s.n_tiles) + size_t(da_slabs(rows, s.S, G)) * s.S) * G * kDc * 4;
}

// da from the partial sums (`partial` at the start of the da_bytes region).
pararnn_status da_reduce(float* partial, float* da, const Shape& s, int G, cudaStream_t stream)
{
    const long long rows = s.B * s.n_chunks;
    const int slabs = da_slabs(rows, s.S, G);
    float* sums = partial + size_t(s.n_tiles) * G * kDc;
    da_slab_kernel<<<dim3(unsigned(s.S * G), unsigned(slabs)), kDc, 0, stream>>>(partial, sums, int(rows), slabs,
                                                                                 s.S * G);
    CUDA_TRY(cudaGetLastError());
    const long long GD = (long long)G * s.D;
    da_final_kernel<<<unsigned((GD + 255) / 256), 256, 0, stream>>>(sums, da, slabs, s.S, G, s.D);
    CUDA_TRY(cudaGetLastError());
    g_launches.fetch_add(2, std::memory_order_relaxed);
    return PARARNN_OK;
}

size_t adjoint_ws_bytes(int cell, long long B, long long L, long long D)
{
    if (!shape_ok(B, L, D) || D % 8 != 0) return 0;
    Shape s;
    char saved[sizeof(t_err)];
    memcpy(saved, t_err, sizeof(t_err));
    pararnn_status st = make_shape(B, L, D, cell == 0 ? adj_lc_min<GruCell>() : adj_lc_min<LstmCell>(), &s);
    memcpy(t_err, saved, sizeof(t_err));
    if (st != PARARNN_OK) return 0;
    const int G = cell == 0 ? 3 : 4;
    const int desc = cell == 0 ? TileDesc<Aff<1>, 1, false>::words : TileDesc<Aff<2>, 2, false>::words;
    return scan_layout(s, desc, da_bytes(s, G)).total;
}

template <class Cell, class UT, int NG = Cell::NS>
pararnn_status launch_adjoint(Shape s, const void* u, pararnn_dtype dt, const float* a, const float* const s0[2],
                              const float* const st[2], const float* const g[2], float* du, float* da,
                              float* const ds0[2], void* ws, cudaStream_t stream)
{
    constexpr int CW = adj_warps<Cell, UT, NG>();
    using LY = AdjointWsLayout<Cell, UT, CW, NG>;
    constexpr int NS = Cell::NS, G = Cell::G;
    TRY(make_shape(s.B, s.L, s.D, LY::Lc, &s));
    const ScanLayout ly = scan_layout(s, LY::desc_words, da_bytes(s, G));
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    CUDA_TRY(cudaMemsetAsync(ws, 0, ly.extra, stream));

    CUtensorMap tu, t0, t1, tg0, tg1;
    TRY(map_gates(&tu, u, dt, G, G, s, LY::Lc));
    TRY(map_state(&t0, st[0], s, LY::Lc + 1));  // from the row before the tile
    TRY(map_state(&t1, st[NS - 1], s, LY::Lc + 1));
    const float* gfirst = g[0] ? g[0] : g[NS - 1];
    TRY(map_state(&tg0, gfirst, s, LY::Lc));
    TRY(map_state(&tg1, g[NS - 1], s, LY::Lc));

    AdjointParams p;
    p.a = a;
    p.s0[0] = s0[0];
    p.s0[1] = s0[1];
    p.st[0] = st[0];
    p.st[1] = st[1];
    p.du = du;
    p.ds0[0] = ds0[0];
    p.ds0[1] = ds0[1];
    p.B = s.B;
    p.L = s.L;
    p.D = s.D;
    p.S = s.S;
    p.n_chunks = s.n_chunks;
    p.n_tiles = s.n_tiles;
    p.has_g[0] = g[0] != nullptr;
    p.has_g[1] = g[1] != nullptr;
    p.hdr = reinterpret_cast<WsHeader*>(wsb);
    p.desc = reinterpret_cast<unsigned long long*>(wsb + ly.desc);
    p.partial = reinterpret_cast<float*>(wsb + ly.extra);
    p.wait_ns = kWaitLimitNs;

    auto kern = adjoint_ws_kernel<Cell, UT, CW, NG>;
    int grid = 0;
    TRY(resident_grid(kern, LY::smem_bytes, s.n_tiles, &grid, LY::threads));
    kern<<<grid, LY::threads, LY::smem_bytes, stream>>>(tu, t0, t1, tg0, tg1, p);
    CUDA_TRY(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return da_reduce(p.partial, da, s, G, stream);
}

pararnn_status adjoint_async(int cell, const void* u, pararnn_dtype dt, const float* a, const float* c0,
                             const float* h0, const float* c, const float* h, const float* dc, const float* dh,
                             float* du, float* da, float* dc0, float* dh0, long long B, long long L, long long D,
                             void* ws, size_t ws_bytes, cudaStream_t stream)
{
    t_err[0] = '\0';
    TRY(check_dtype(dt));
    TRY(check_ptr(u, "u", true));
    TRY(check_ptr(a, "a", true));
    TRY(check_ptr(h0, "h0", false));
    TRY(check_ptr(h, "h", true));
    TRY(check_ptr(dh, "dh", true));
    TRY(check_ptr(du, "du", true));
    TRY(check_ptr(da, "da", true));
    TRY(check_ptr(dh0, "dh0", false));
    if (cell == 1) {
        TRY(check_ptr(c0, "c0", false));
        TRY(check_ptr(c, "c", true));
        TRY(check_ptr(dc, "dc", false));
        TRY(check_ptr(dc0, "dc0", false));
    }
    Shape s;
    TRY(make_shape(B, L, D, cell == 0 ? adj_lc_min<GruCell>() : adj_lc_min<LstmCell>(), &s));
    TRY(check_workspace(ws, ws_bytes, adjoint_ws_bytes(cell, B, L, D)));
    if (cell == 0) {
        const float* s0[2] = {h0, nullptr};
        const float* st[2] = {h, nullptr};
        const float* g[2] = {dh, nullptr};
        float* ds0[2] = {dh0, nullptr};
        if (dt == PARARNN_BF16)
            return launch_adjoint<GruCell, uint16_t>(s, u, dt, a, s0, st, g, du, da, ds0, ws, stream);
        return launch_adjoint<GruCell, float>(s, u, dt, a, s0, st, g, du, da, ds0, ws, stream);
    }
    const float* s0[2] = {c0, h0};
    const float* st[2] = {c, h};
    const float* g[2] = {dc, dh};
    float* ds0[2] = {dc0, dh0};
    if (!dc) {  // a loss on h alone: one upstream component staged
        if (dt == PARARNN_BF16)
            return launch_adjoint<LstmCell, uint16_t, 1>(s, u, dt, a, s0, st, g, du, da, ds0, ws, stream);
        return launch_adjoint<LstmCell, float, 1>(s, u, dt, a, s0, st, g, du, da, ds0, ws, stream);
    }
    if (dt == PARARNN_BF16)
        return launch_adjoint<LstmCell, uint16_t>(s, u, dt, a, s0, st, g, du, da, ds0, ws, stream);
    return launch_adjoint<LstmCell, float>(s, u, dt, a, s0, st, g, du, da, ds0, ws, stream);
}

// ------------------------------------------------------------ linear scan

// bf16 gates: 15 compute warps of 4 steps (60-step tiles; with the control
// warp, 16 warps of up to 128 registers); fp32 gates take
// twice the staging space, so their warps take 2 steps
#ifndef PARARNN_LIN_CW
#define PARARNN_LIN_CW 15
#endif
constexpr int kLinWarps = PARARNN_LIN_CW;
template <class UT> constexpr int lin_rows() { return sizeof(UT) == 2 ? 4 : 2; }
template <class UT> constexpr int lin_lc() { return kLinWarps * lin_rows<UT>(); }

size_t linear_scan_ws_bytes(long long B, long long L, long long D)
{
    if (!shape_ok(B, L, D) || D % 8 != 0) return 0;
    Shape s;
    char saved[sizeof(t_err)];
    memcpy(saved, t_err, sizeof(t_err));
    pararnn_status st = make_shape(B, L, D, lin_lc<float>(), &s);  // the shorter tile: more groups
    memcpy(t_err, saved, sizeof(t_err));
    if (st != PARARNN_OK) return 0;
    return scan_layout(s, LinScanLayout<float, kLinWarps, lin_rows<float>()>::desc_words, 0, solve_descs(s)).total;
}

// Whether the linear scan's look-backs step back over aggregates.
#ifndef PARARNN_LIN_WALK
#define PARARNN_LIN_WALK -1  // -1: chosen from the shape
#endif
int linear_scan_walks(int grid, long long sequences)
{
    return PARARNN_LIN_WALK >= 0 ? PARARNN_LIN_WALK : solve_lookback_walks(grid, sequences);
}

template <class UT>
pararnn_status launch_linear_scan(const void* u, pararnn_dtype dt, const float* h0, float* h, long long B,
                                  long long L, long long D, void* ws, cudaStream_t stream)
{
    constexpr int R = lin_rows<UT>();
    using LY = LinScanLayout<UT, kLinWarps, R>;
    Shape s;
    TRY(make_shape(B, L, D, LY::Lc, &s));
    const ScanLayout ly = scan_layout(s, LY::desc_words, 0, solve_descs(s));
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    CUDA_TRY(cudaMemsetAsync(ws, 0, ly.extra, stream));
    CUtensorMap tu;
    TRY(map_gates(&tu, u, dt, 3, 1, s, LY::Lc));
    LinScanParams p;
    p.h0 = h0;
    p.h = h;
    p.B = s.B;
    p.L = s.L;
    p.D = s.D;
    p.S = s.S;
    p.n_chunks = s.n_chunks;
    p.n_tiles = s.n_tiles;
    p.hdr = reinterpret_cast<WsHeader*>(wsb);
    p.desc = reinterpret_cast<unsigned long long*>(wsb + ly.desc);
    p.wait_ns = kWaitLimitNs;
    auto kern = linear_scan_kernel<UT, kLinWarps, R>;
    int grid = 0;
    TRY(resident_grid(kern, LY::smem_bytes, int(solve_descs(s)), &grid, LY::threads));
    p.lb_walk = linear_scan_walks(grid, s.B * s.S);
    kern<<<grid, LY::threads, LY::smem_bytes, stream>>>(tu, p);
    CUDA_TRY(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PARARNN_OK;
}

pararnn_status linear_scan_async(const void* u, pararnn_dtype dt, const float* h0, float* h, long long B, long long L,
                                 long long D, void* ws, size_t ws_bytes, cudaStream_t stream)
{
    t_err[0] = '\0';
    TRY(check_dtype(dt));
    TRY(check_ptr(u, "u", true));
    TRY(check_ptr(h0, "h0", false));
    TRY(check_ptr(h, "h", true));
    Shape s;
    TRY(make_shape(B, L, D, lin_lc<float>(), &s));
    TRY(check_workspace(ws, ws_bytes, linear_scan_ws_bytes(B, L, D)));
    if (dt == PARARNN_BF16) return launch_linear_scan<uint16_t>(u, dt, h0, h, B, L, D, ws, stream);
    return launch_linear_scan<float>(u, dt, h0, h, B, L, D, ws, stream);
}

// -------------------------------------------------------------- self tests

pararnn_status selftest_wait_timeout(int which, long long limit_ns, void* ws, size_t ws_bytes, cudaStream_t stream)
{
    t_err[0] = '\0';
    if (which != 0 && which != 1) return fail(PARARNN_ERR_INVALID_ARG, "which must be 0 or 1");
    if (limit_ns <= 0 || limit_ns > 10000000000ll) return fail(PARARNN_ERR_INVALID_ARG, "limit_ns out of range");
    TRY(check_workspace(ws, ws_bytes, kSelftestWorkspace));
    CUDA_TRY(cudaMemsetAsync(ws, 0, kSelftestWorkspace, stream));
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(wsb);
    unsigned long long* desc = reinterpret_cast<unsigned long long*>(wsb + sizeof(WsHeader));
    unsigned long long lim = (unsigned long long)limit_ns;
    if (which == 0) {
        selftest_lookback_kernel<<<1, 32, 0, stream>>>(desc, &hdr->error, lim);
        CUDA_TRY(cudaGetLastError());
    } else {
        int sms = 0;
        TRY(device_info(&sms));
        unsigned* counter = &hdr->bar;
        int* err = &hdr->error;
        void* args[] = {(void*)&counter, (void*)&err, (void*)&lim};
        CUDA_TRY(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(selftest_barrier_kernel), dim3(2), dim3(32),
                                             args, 0, stream));
    }
    g_launches.fetch_add(1, std::memory_order_relaxed);
    WsHeader h;
    TRY(read_header(ws, stream, &h));
    if (h.error != 0) return fail(pararnn_status(h.error), "bounded wait gave up as expected");
    return PARARNN_OK;
}

// ------------------------------------------------ fixed scratch (no-alloc)
//
// Scratch of pararnn_gru_solve_noalloc: one array per device, part of this
// library's module image, so using it needs no allocation call at all.  Its
// address is looked up once per device (cudaGetSymbolAddress, with that
// device current) and cached.  Calls that overlap in time on one device
// share it and race.

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kNoAllocMaxDevices = 64;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

pararnn_status noalloc_scratch(void** out)
{
    int dev = -1;
    CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(PARARNN_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || !ptr)
            return fail(PARARNN_ERR_CUDA, "cudaGetSymbolAddress(scratch) on device %d: %s", dev, cudaGetErrorString(e));
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return PARARNN_OK;
}

// decode step: shape and aliasing checks, launch
pararnn_status check_step_shape(int64_t B, int64_t D)
{
    if (B < 1 || D < 1) return fail(PARARNN_ERR_INVALID_ARG, "B, D must be >= 1 (got %lld, %lld)", (long long)B,
                                    (long long)D);
    if (D % 8 != 0) return fail(PARARNN_ERR_UNSUPPORTED, "D must be a multiple of 8 (got %lld)", (long long)D);
    if ((double)B * (double)D * 16.0 >= 1099511627776.0) return fail(PARARNN_ERR_INVALID_ARG, "B*D too large");
    return PARARNN_OK;
}

// do the n-float ranges at x and y share a byte?
bool overlap(const float* x, const float* y, long long n)
{
    if (!x || !y) return false;
    const uintptr_t x0 = reinterpret_cast<uintptr_t>(x), y0 = reinterpret_cast<uintptr_t>(y);
    const uintptr_t len = uintptr_t(n) * 4;
    return x0 < y0 + len && y0 < x0 + len;
}

// an output may be its own previous state; any other overlap is refused
pararnn_status check_alias(const float* in, const float* out, long long n, const char* name)
{
    if (in != out && overlap(in, out, n))
        return fail(PARARNN_ERR_INVALID_ARG, "%s overlaps an input without being its own previous state", name);
    return PARARNN_OK;
}

template <class Cell>
pararnn_status launch_step(const void* u, pararnn_dtype u_dtype, const float* a, const float* p0, const float* p1,
                           float* n0, float* n1, int64_t B, int64_t D, cudaStream_t st)
{
    const long long n4 = (long long)B * D / 4;
    if (n4 == 0) return PARARNN_OK;
    const dim3 block(256), grid(unsigned((n4 + 255) / 256));
    if (u_dtype == PARARNN_BF16)
        decode_step_kernel<Cell, uint16_t>
            <<<grid, block, 0, st>>>(static_cast<const uint16_t*>(u), a, p0, p1, n0, n1, B, D);
    else
        decode_step_kernel<Cell, float><<<grid, block, 0, st>>>(static_cast<const float*>(u), a, p0, p1, n0, n1, B, D);
    CUDA_TRY(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PARARNN_OK;
}

}  // namespace

// =================================================================== C ABI

extern "C" {

size_t pararnn_gru_workspace_size(int64_t B, int64_t L, int64_t D) { return solve_ws_bytes(0, B, L, D); }
size_t pararnn_lstm_workspace_size(int64_t B, int64_t L, int64_t D) { return solve_ws_bytes(1, B, L, D); }

pararnn_status pararnn_gru_solve_async(const void* u, pararnn_dtype u_dtype, const float* a, const float* h0, float* h,
                                       int64_t B, int64_t L, int64_t D, float tol, int max_iters, void* workspace,
                                       size_t workspace_bytes, pararnn_stream_t stream)
{
    return solve_async(0, u, u_dtype, a, nullptr, h0, nullptr, h, B, L, D, tol, max_iters, workspace,
                       workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

pararnn_status pararnn_gru_solve(const void* u, pararnn_dtype u_dtype, const float* a, const float* h0, float* h,
                                 int64_t B, int64_t L, int64_t D, float tol, int max_iters, void* workspace,
                                 size_t workspace_bytes, pararnn_stream_t stream, int* iters_out, float* residual_out)
{
    TRY(pararnn_gru_solve_async(u, u_dtype, a, h0, h, B, L, D, tol, max_iters, workspace, workspace_bytes, stream));
    return finish_sync(workspace, reinterpret_cast<cudaStream_t>(stream), iters_out, residual_out);
}

pararnn_status pararnn_gru_solve_noalloc(const void* u, pararnn_dtype u_dtype, const float* a, const float* h0,
                                         float* h, int64_t B, int64_t L, int64_t D, float tol, int max_iters,
                                         pararnn_stream_t stream, int* iters_out, float* residual_out)
{
    t_err[0] = '\0';
    // every argument check happens here, on the host, before the scratch
    // lookup (which is the first device call)
    TRY(solve_args(0, u, u_dtype, a, nullptr, h0, nullptr, h, B, L, D, tol, max_iters));
    const size_t need = pararnn_gru_workspace_size(B, L, D);
    if (need > kNoAllocScratchBytes)
        return fail(PARARNN_ERR_WORKSPACE,
                    "B=%lld L=%lld D=%lld needs %zu bytes of scratch; the fixed scratch holds %zu "
                    "(use pararnn_gru_solve with a caller workspace)",
                    (long long)B, (long long)L, (long long)D, need, kNoAllocScratchBytes);
    void* ws = nullptr;
    TRY(noalloc_scratch(&ws));
    // the solve itself zeroes the scratch's header and tile descriptors on
    // the stream before its kernel runs (as it does for any workspace)
    return pararnn_gru_solve(u, u_dtype, a, h0, h, B, L, D, tol, max_iters, ws, kNoAllocScratchBytes, stream,
                             iters_out, residual_out);
}

size_t pararnn_gru_solve_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

size_t pararnn_gru_project_workspace_size(int64_t B, int64_t L, int64_t D, int64_t Din)
{
    return project_ws_bytes(B, L, D, Din);
}

pararnn_status pararnn_gru_project_solve_async(const void* x, const void* w, const float* bias, const float* a,
                                               const float* h0, void* u, float* h, int64_t B, int64_t L,
                                               int64_t Din, int64_t D, float tol, int max_iters, void* workspace,
                                               size_t workspace_bytes, pararnn_stream_t stream)
{
    return project_solve_async(x, w, bias, a, h0, static_cast<uint16_t*>(u), h, B, L, Din, D, tol, max_iters,
                               workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

pararnn_status pararnn_gru_project_solve(const void* x, const void* w, const float* bias, const float* a,
                                         const float* h0, void* u, float* h, int64_t B, int64_t L, int64_t Din,
                                         int64_t D, float tol, int max_iters, void* workspace,
                                         size_t workspace_bytes, pararnn_stream_t stream, int* iters_out,
                                         float* residual_out)
{
    TRY(pararnn_gru_project_solve_async(x, w, bias, a, h0, u, h, B, L, Din, D, tol, max_iters, workspace,
                                        workspace_bytes, stream));
    return finish_sync(workspace, reinterpret_cast<cudaStream_t>(stream), iters_out, residual_out);
}

pararnn_status pararnn_lstm_solve_async(const void* u, pararnn_dtype u_dtype, const float* a, const float* c0,
                                        const float* h0, float* c, float* h, int64_t B, int64_t L, int64_t D,
                                        float tol, int max_iters, void* workspace, size_t workspace_bytes,
                                        pararnn_stream_t stream)
{
    return solve_async(1, u, u_dtype, a, c0, h0, c, h, B, L, D, tol, max_iters, workspace, workspace_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

pararnn_status pararnn_lstm_solve(const void* u, pararnn_dtype u_dtype, const float* a, const float* c0,
                                  const float* h0, float* c, float* h, int64_t B, int64_t L, int64_t D, float tol,
                                  int max_iters, void* workspace, size_t workspace_bytes, pararnn_stream_t stream,
                                  int* iters_out, float* residual_out)
{
    TRY(pararnn_lstm_solve_async(u, u_dtype, a, c0, h0, c, h, B, L, D, tol, max_iters, workspace, workspace_bytes,
                                 stream));
    return finish_sync(workspace, reinterpret_cast<cudaStream_t>(stream), iters_out, residual_out);
}

pararnn_status pararnn_read_pass_times(const void* workspace, pararnn_stream_t stream, double* pass_us, int max_passes,
                                       int* n_passes)
{
    t_err[0] = '\0';
    if (max_passes < 0 || (max_passes > 0 && !pass_us)) return fail(PARARNN_ERR_INVALID_ARG, "pass_us is NULL");
    WsHeader h;
    TRY(read_header(workspace, reinterpret_cast<cudaStream_t>(stream), &h));
    int n = 0;
    while (n + 1 < kPassTimes && h.t_pass[n + 1] != 0 && h.t_pass[n + 1] >= h.t_pass[n]) ++n;
    if (h.t_pass[0] == 0) n = 0;
    for (int i = 0; i < n && i < max_passes; ++i) pass_us[i] = double(h.t_pass[i + 1] - h.t_pass[i]) * 1e-3;
    if (n_passes) *n_passes = n;
    return PARARNN_OK;
}

pararnn_status pararnn_read_result(const void* workspace, pararnn_stream_t stream, pararnn_result* result)
{
    WsHeader h;
    TRY(read_header(workspace, reinterpret_cast<cudaStream_t>(stream), &h));
    pararnn_result r = h.result;
    if (h.error != 0) {
        r.status = h.error;
        fail(pararnn_status(h.error), "device-side error %d (%s)", h.error, pararnn_status_string(pararnn_status(h.error)));
    }
    if (result) *result = r;
    return pararnn_status(r.status);
}

pararnn_status pararnn_result_to_device(const void* workspace, float* out, pararnn_stream_t stream)
{
    t_err[0] = '\0';
    if (!workspace) return fail(PARARNN_ERR_WORKSPACE, "workspace is NULL");
    if (!out) return fail(PARARNN_ERR_INVALID_ARG, "out is NULL");
    result_outcome_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const WsHeader*>(workspace), out);
    CUDA_TRY(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PARARNN_OK;
}

// ------------------------------------------------------------- adjoints

size_t pararnn_gru_adjoint_workspace_size(int64_t B, int64_t L, int64_t D) { return adjoint_ws_bytes(0, B, L, D); }
size_t pararnn_lstm_adjoint_workspace_size(int64_t B, int64_t L, int64_t D) { return adjoint_ws_bytes(1, B, L, D); }

pararnn_status pararnn_gru_adjoint(const void* u, pararnn_dtype u_dtype, const float* a, const float* h0,
                                   const float* h, const float* dh, float* du, float* da, float* dh0, int64_t B,
                                   int64_t L, int64_t D, void* workspace, size_t workspace_bytes,
                                   pararnn_stream_t stream)
{
    return adjoint_async(0, u, u_dtype, a, nullptr, h0, nullptr, h, nullptr, dh, du, da, nullptr, dh0, B, L, D,
                         workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

pararnn_status pararnn_lstm_adjoint(const void* u, pararnn_dtype u_dtype, const float* a, const float* c0,
                                    const float* h0, const float* c, const float* h, const float* dh, const float* dc,
                                    float* du, float* da, float* dc0, float* dh0, int64_t B, int64_t L, int64_t D,
                                    void* workspace, size_t workspace_bytes, pararnn_stream_t stream)
{
    return adjoint_async(1, u, u_dtype, a, c0, h0, c, h, dc, dh, du, da, dc0, dh0, B, L, D, workspace,
                         workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------- baselines

pararnn_status pararnn_gru_sequential(const void* u, pararnn_dtype u_dtype, const float* a, const float* h0, float* h,
                                      int64_t B, int64_t L, int64_t D, pararnn_stream_t stream)
{
    t_err[0] = '\0';
    TRY(check_dtype(u_dtype));
    TRY(check_ptr(u, "u", true));
    TRY(check_ptr(a, "a", true));
    TRY(check_ptr(h0, "h0", false));
    TRY(check_ptr(h, "h", true));
    Shape s;
    TRY(make_shape(B, L, D, 1, &s));
    const long long n = B * D;
    const dim3 grid(unsigned((n + 63) / 64)), block(64);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (u_dtype == PARARNN_BF16)
        sequential_kernel<GruCell, uint16_t><<<grid, block, 0, st>>>(static_cast<const uint16_t*>(u), a, h0, nullptr,
                                                                     h, nullptr, B, L, D);
    else
        sequential_kernel<GruCell, float><<<grid, block, 0, st>>>(static_cast<const float*>(u), a, h0, nullptr, h,
                                                                  nullptr, B, L, D);
    CUDA_TRY(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PARARNN_OK;
}

pararnn_status pararnn_lstm_sequential(const void* u, pararnn_dtype u_dtype, const float* a, const float* c0,
                                       const float* h0, float* c, float* h, int64_t B, int64_t L, int64_t D,
                                       pararnn_stream_t stream)
{
    t_err[0] = '\0';
    TRY(check_dtype(u_dtype));
    TRY(check_ptr(u, "u", true));
    TRY(check_ptr(a, "a", true));
    TRY(check_ptr(c0, "c0", false));
    TRY(check_ptr(h0, "h0", false));
    TRY(check_ptr(c, "c", true));
    TRY(check_ptr(h, "h", true));
    Shape s;
    TRY(make_shape(B, L, D, 1, &s));
    const long long n = B * D;
    const dim3 grid(unsigned((n + 63) / 64)), block(64);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (u_dtype == PARARNN_BF16)
        sequential_kernel<LstmCell, uint16_t><<<grid, block, 0, st>>>(static_cast<const uint16_t*>(u), a, c0, h0, c,
                                                                      h, B, L, D);
    else
        sequential_kernel<LstmCell, float><<<grid, block, 0, st>>>(static_cast<const float*>(u), a, c0, h0, c, h, B,
                                                                   L, D);
    CUDA_TRY(cudaGetLastError());
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PARARNN_OK;
}

// ---------------------------------------------------------- decode step

pararnn_status pararnn_gru_step(const void* u, pararnn_dtype u_dtype, const float* a, const float* h_prev,
                                float* h_next, int64_t B, int64_t D, pararnn_stream_t stream)
{
    t_err[0] = '\0';
    TRY(check_dtype(u_dtype));
    TRY(check_ptr(u, "u", true));
    TRY(check_ptr(a, "a", true));
    TRY(check_ptr(h_prev, "h_prev", false));
    TRY(check_ptr(h_next, "h_next", true));
    TRY(check_step_shape(B, D));
    TRY(check_alias(h_prev, h_next, (long long)B * D, "h_next"));
    return launch_step<GruCell>(u, u_dtype, a, h_prev, nullptr, h_next, nullptr, B, D,
                                reinterpret_cast<cudaStream_t>(stream));
}

pararnn_status pararnn_lstm_step(const void* u, pararnn_dtype u_dtype, const float* a, const float* c_prev,
                                 const float* h_prev, float* c_next, float* h_next, int64_t B, int64_t D,
                                 pararnn_stream_t stream)
{
    t_err[0] = '\0';
    TRY(check_dtype(u_dtype));
    TRY(check_ptr(u, "u", true));
    TRY(check_ptr(a, "a", true));
    TRY(check_ptr(c_prev, "c_prev", false));
    TRY(check_ptr(h_prev, "h_prev", false));
    TRY(check_ptr(c_next, "c_next", true));
    TRY(check_ptr(h_next, "h_next", true));
    TRY(check_step_shape(B, D));
    const long long n = (long long)B * D;
    TRY(check_alias(c_prev, c_next, n, "c_next"));
    TRY(check_alias(h_prev, h_next, n, "h_next"));
    if (overlap(h_prev, c_next, n)) return fail(PARARNN_ERR_INVALID_ARG, "c_next overlaps h_prev");
    if (overlap(c_prev, h_next, n)) return fail(PARARNN_ERR_INVALID_ARG, "h_next overlaps c_prev");
    if (overlap(c_next, h_next, n)) return fail(PARARNN_ERR_INVALID_ARG, "c_next and h_next overlap");
    return launch_step<LstmCell>(u, u_dtype, a, c_prev, h_prev, c_next, h_next, B, D,
                                 reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------- segments of a sequence

pararnn_status pararnn_gru_segment_pass(const void* u, pararnn_dtype u_dtype, const float* a, const float* h_in,
                                        const float* h_lin, const float* h_carry, float* h_out, float* h_end,
                                        int64_t B, int64_t L, int64_t D, void* workspace, size_t workspace_bytes,
                                        pararnn_stream_t stream)
{
    return segment_pass_async(0, u, u_dtype, a, h_in, h_lin, h_carry, h_out, h_end, B, L, D, workspace,
                              workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

pararnn_status pararnn_lstm_segment_pass(const void* u, pararnn_dtype u_dtype, const float* a, const float* s_in,
                                         const float* s_lin, const float* s_carry, float* s_out, float* s_end,
                                         int64_t B, int64_t L, int64_t D, void* workspace, size_t workspace_bytes,
                                         pararnn_stream_t stream)
{
    return segment_pass_async(1, u, u_dtype, a, s_in, s_lin, s_carry, s_out, s_end, B, L, D, workspace,
                              workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t pararnn_segment_record_floats(int n_state, int64_t B, int64_t D)
{
    if ((n_state != 1 && n_state != 2) || B < 1 || D < 1) return 0;
    return size_t(segment_record_floats(n_state - 1, (long long)B * D));
}

size_t pararnn_segment_fold_workspace_size(int n_state, int64_t B, int64_t L, int64_t D)
{
    if (n_state != 1 && n_state != 2) return 0;
    return segment_fold_ws_bytes(n_state - 1, B, L, D);
}

pararnn_status pararnn_gru_segment_fold(const void* u, pararnn_dtype u_dtype, const float* a, const float* h_in,
                                        float* record, int64_t B, int64_t L, int64_t D, void* workspace,
                                        size_t workspace_bytes, pararnn_stream_t stream)
{
    return segment_fold_async(0, u, u_dtype, a, h_in, record, B, L, D, workspace, workspace_bytes,
                              reinterpret_cast<cudaStream_t>(stream));
}

pararnn_status pararnn_lstm_segment_fold(const void* u, pararnn_dtype u_dtype, const float* a, const float* s_in,
                                         float* record, int64_t B, int64_t L, int64_t D, void* workspace,
                                         size_t workspace_bytes, pararnn_stream_t stream)
{
    return segment_fold_async(1, u, u_dtype, a, s_in, record, B, L, D, workspace, workspace_bytes,
                              reinterpret_cast<cudaStream_t>(stream));
}

pararnn_status pararnn_gru_segment_combine(const float* records, int n_segments, int index, const float* a,
                                           const float* h0, float* h_carry, float* h_lin, float* residual, int64_t B,
                                           int64_t D, pararnn_stream_t stream)
{
    return segment_combine_async(0, records, n_segments, index, a, h0, h_carry, h_lin, residual, B, D,
                                 reinterpret_cast<cudaStream_t>(stream));
}

pararnn_status pararnn_lstm_segment_combine(const float* records, int n_segments, int index, const float* a,
                                            const float* s0, float* s_carry, float* s_lin, float* residual,
                                            int64_t B, int64_t D, pararnn_stream_t stream)
{
    return segment_combine_async(1, records, n_segments, index, a, s0, s_carry, s_lin, residual, B, D,
                                 reinterpret_cast<cudaStream_t>(stream));
}

size_t pararnn_linear_scan_workspace_size(int64_t B, int64_t L, int64_t D) { return linear_scan_ws_bytes(B, L, D); }

pararnn_status pararnn_linear_scan(const void* u, pararnn_dtype u_dtype, const float* h0, float* h, int64_t B,
                                   int64_t L, int64_t D, void* workspace, size_t workspace_bytes,
                                   pararnn_stream_t stream)
{
    return linear_scan_async(u, u_dtype, h0, h, B, L, D, workspace, workspace_bytes,
                             reinterpret_cast<cudaStream_t>(stream));
}

// ----------------------------------------------------------- diagnostics

const char* pararnn_status_string(pararnn_status s)
{
    switch (s) {
    case PARARNN_OK: return "ok";
    case PARARNN_NOT_CONVERGED: return "not converged";
    case PARARNN_ERR_INVALID_ARG: return "invalid argument";
    case PARARNN_ERR_WORKSPACE: return "workspace missing or too small";
    case PARARNN_ERR_CUDA: return "CUDA error";
    case PARARNN_ERR_TIMEOUT: return "device-side wait timed out";
    case PARARNN_ERR_NONFINITE: return "non-finite residual";
    case PARARNN_ERR_UNSUPPORTED: return "unsupported";
    }
    return "unknown status";
}

const char* pararnn_last_error(void) { return t_err; }

const char* pararnn_version(void) { return "0.1.0"; }

uint64_t pararnn_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

pararnn_status pararnn_selftest_wait_timeout(int which, int64_t limit_ns, void* workspace, size_t workspace_bytes,
                                             pararnn_stream_t stream)
{
    return selftest_wait_timeout(which, limit_ns, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// user-written cells, compiled at run time
#include "cell_rtc_host.h"
