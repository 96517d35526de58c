// The parts of the chunked parallel scan of affine maps that the Newton
// solve, the adjoint and the linear-scan baseline share: the tagged words
// through which tiles hand values to one another, and the look-back.
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros", section "O compromisso que SSMs fizeram": a linear
// recurrence is an associative combination, so it can be evaluated as a tree
// (O(log L) depth) instead of step by step; section "A sacada: método de
// Newton": every Newton iteration is such a linear recurrence.
//
// Every scan kernel works in three levels: (1) each compute warp folds the
// maps of its two steps of a tile in registers; (2) the CTA's control warp
// composes the warps' folds into exclusive prefixes; (3) tiles (or groups of
// tiles) are chained across CTAs: each publishes its aggregate, resolves the
// value entering it from its predecessors' published words (stepping back
// over aggregates, or waiting for the predecessor's inclusive value), and
// publishes its inclusive value.  Values travel as tagged 64-bit words (each
// word is its own ready flag, so no fences); every wait is bounded.
#pragma once

#include "cells.cuh"

namespace pararnn {

// Published values are tagged 64-bit words: the float in the low half, a tag
// in the high half.  An aligned 64-bit access is single-copy atomic, so a
// reader that sees the expected tag also sees the value written with it: the
// word is its own flag, and neither side needs a fence.  Tags are 2*epoch+1
// (tile aggregate) and 2*epoch+2 (inclusive value); the words are zeroed
// before each launch, and tags only grow within a launch.
__device__ __forceinline__ unsigned long long tag_word(float v, unsigned tag)
{
    return (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(v);
}

__device__ __forceinline__ void st_words2(unsigned long long* p, unsigned long long a, unsigned long long b)
{
    asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}

__device__ __forceinline__ void ld_words2(const unsigned long long* p, unsigned long long& a, unsigned long long& b)
{
    asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

// Descriptor of one tile (or group of tiles) in the workspace, in tagged
// words: aggregates [32 lanes][kV * NC], then inclusive values
// [32 lanes][kV * NS].  Agg = false drops the aggregates, for look-backs that
// only ever wait for inclusive values: the descriptors are then a third
// (ParaGRU) or a quarter (ParaLSTM) as large, and so is their zeroing.
template <class Map, int NS, bool Agg = true>
struct TileDesc {
    static constexpr int agg_words = Agg ? 32 * kV * Map::kFloats : 0;
    static constexpr int words = agg_words + 32 * kV * NS;
};

// Store n (even) tagged words.
template <int N>
__device__ __forceinline__ void publish_words(unsigned long long* dst, const float (&v)[N], unsigned tag)
{
    static_assert(N % 2 == 0, "pairs");
#pragma unroll
    for (int i = 0; i < N; i += 2) st_words2(dst + i, tag_word(v[i], tag), tag_word(v[i + 1], tag));
}

// Load n (even) words.
template <int N>
__device__ __forceinline__ void load_words(const unsigned long long* src, unsigned long long (&w)[N])
{
    static_assert(N % 2 == 0, "pairs");
#pragma unroll
    for (int i = 0; i < N; i += 2) ld_words2(src + i, w[i], w[i + 1]);
}

// Values of n loaded words; true if every tag equals `tag`.
template <int N>
__device__ __forceinline__ bool unpack_words(const unsigned long long (&w)[N], float (&v)[N], unsigned tag)
{
    bool ok = true;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        ok = ok && unsigned(w[i] >> 32) == tag;
        v[i] = __uint_as_float(unsigned(w[i]));
    }
    return ok;
}

// First look-back probe: the words of the predecessor tile (its inclusive
// value and its aggregate), loaded early so that the round trip overlaps
// whatever the caller does before calling lookback_resolve().
template <class Map, int NS>
struct LookbackProbe {
    unsigned long long wi[kV * NS];
    unsigned long long wa[kV * Map::kFloats];
};

// (WithAgg = false: the inclusive value only, for a look-back that waits for
// it instead of stepping back.)
template <class Map, int NS, bool WithAgg = true, class TD = TileDesc<Map, NS>>
__device__ __forceinline__ void lookback_probe(LookbackProbe<Map, NS>& pr, int pred_ticket,
                                               const unsigned long long* desc, int lane)
{
    static_assert(!WithAgg || TD::agg_words > 0, "descriptors without aggregates");
    const unsigned long long* pd = desc + (size_t)pred_ticket * TD::words;
    load_words(pd + TD::agg_words + lane * kV * NS, pr.wi);
    if (WithAgg) load_words(pd + lane * kV * Map::kFloats, pr.wa);
}

// Publish maps (a tile's or a group's aggregate) under tag 2*epoch+1.
template <class Map, int NS, class TD = TileDesc<Map, NS>>
__device__ __forceinline__ void publish_aggregate(unsigned long long* desc, int ticket, int epoch, const Map (&ta)[kV],
                                                  int lane)
{
    static_assert(TD::agg_words > 0, "descriptors without aggregates");
    constexpr int NC = Map::kFloats;
    float av[kV * NC];
#pragma unroll
    for (int j = 0; j < kV; ++j)
#pragma unroll
        for (int i = 0; i < NC; ++i) av[j * NC + i] = ta[j].get(i);
    publish_words(desc + (size_t)ticket * TD::words + lane * kV * NC, av, 2u * epoch + 1u);
}

// Publish an inclusive value (the state leaving a tile or group) under tag
// 2*epoch+2.
template <class Map, int NS, class TD = TileDesc<Map, NS>>
__device__ __forceinline__ void publish_inclusive(unsigned long long* desc, int ticket, int epoch,
                                                  const float (&incl)[NS][kV], int lane)
{
    float iv[kV * NS];
#pragma unroll
    for (int j = 0; j < kV; ++j)
#pragma unroll
        for (int q = 0; q < NS; ++q) iv[j * NS + q] = incl[q][j];
    publish_words(desc + (size_t)ticket * TD::words + TD::agg_words + lane * kV * NS, iv, 2u * epoch + 2u);
}

// Decoupled look-back, run by one full warp; lane owns channels lane*kV..+kV-1.
// Resolves the value entering tile `ticket` (whose predecessor is
// ticket - stride) from its predecessors' descriptors:
//   epoch:     tags 2*epoch+1 (aggregate), 2*epoch+2 (inclusive)
//   carry:     out: value entering this tile (the predecessors' inclusive)
//   pr:        the first probe (lookback_probe of ticket - stride)
//   Walk:      step back over a predecessor that has published only its
//              aggregate (the decoupled look-back); if false, wait for the
//              predecessor's inclusive value instead (a chain of inclusive
//              values, which is faster when few tiles of one sequence are in
//              flight at once) and read no aggregates at all (the probe must
//              then come from lookback_probe<..., false>)
//   TD:        the descriptor layout (aggregate-free only when !Walk)
// Each step back reads the predecessor's inclusive value and aggregate
// together (one round trip).  Each lane walks back on its own; a wait that
// runs out of time raises PARARNN_ERR_TIMEOUT and returns false.
template <class Map, int NS, bool Walk = true, class TD = TileDesc<Map, NS>>
__device__ __forceinline__ bool lookback_resolve(int ticket, int stride, int epoch, float (&carry)[NS][kV],
                                                 const unsigned long long* desc, int lane, int* err,
                                                 unsigned long long wait_ns, LookbackProbe<Map, NS>& pr)
{
    constexpr int NC = Map::kFloats;
    const unsigned t_agg = 2u * epoch + 1u, t_incl = 2u * epoch + 2u;
    bool ok = true;
    Map acc[kV];
#pragma unroll
    for (int j = 0; j < kV; ++j) acc[j] = Map::identity();
    int jt = ticket - stride;
    bool done = false;
    uint64_t t0 = 0;
    unsigned spins = 0;
    while (__any_sync(0xffffffffu, !done)) {
        if (!done) {
            float iv[kV * NS];
            float av[kV * NC];
            if (unpack_words(pr.wi, iv, t_incl)) {
#pragma unroll
                for (int j = 0; j < kV; ++j) {
                    float x[NS], y[NS];
#pragma unroll
                    for (int q = 0; q < NS; ++q) x[q] = iv[j * NS + q];
                    apply(acc[j], x, y);
#pragma unroll
                    for (int q = 0; q < NS; ++q) carry[q][j] = y[q];
                }
                done = true;
            } else if (Walk && unpack_words(pr.wa, av, t_agg)) {
#pragma unroll
                for (int j = 0; j < kV; ++j) {
                    Map e;
#pragma unroll
                    for (int i = 0; i < NC; ++i) e.set(i, av[j * NC + i]);
                    acc[j] = compose(acc[j], e);
                }
                jt -= stride;
                spins = 0;
                lookback_probe<Map, NS, Walk, TD>(pr, jt, desc, lane);  // (Walk is true here)
            } else {
                // predecessor not published yet: back off, bounded
                if ((++spins & 15u) == 0u) {
                    if (error_raised(err)) {
                        ok = false;
                        done = true;
                    } else {
                        const uint64_t now = global_timer_ns();
                        if (t0 == 0) {
                            t0 = now;
                        } else if (now - t0 > wait_ns) {
                            raise_error(err, PARARNN_ERR_TIMEOUT);
                            ok = false;
                            done = true;
                        }
                    }
                }
                if (spins > 32) __nanosleep(64);
                if (!done) lookback_probe<Map, NS, Walk, TD>(pr, jt, desc, lane);
            }
        }
    }
    return __all_sync(0xffffffffu, ok);
}

}  // namespace pararnn
