// Parameters and stopping rule shared by the fused ParaRNN Newton solve
// kernels (newton_ws.cuh).
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros".
//   "A sacada: método de Newton": the unknowns are all states H; iteration k
//     evaluates F_l(H^k) = s_l - f(s_{l-1}, u_l) and J_l = df/ds_{l-1}, and
//     solves the linear SSM delta_l = J_l delta_{l-1} - F_l (delta_0 = 0) by
//     a parallel scan; H^{k+1} = H^k + delta.
//   "Engenharia pra escalar": Newton iterations, system assembly and the
//     parallel reduction fused in one kernel.
// Between iterations every CTA passes a grid barrier, reads the global
// residual maxima and takes the same decision (newton_decide), so the loop
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
    int lb_walk;            // look-backs step over aggregates (many groups of a sequence in flight)
    int skip_res;           // ParaGRU: passes that continue may leave residuals out (many tiles per CTA)
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

}  // namespace pararnn
