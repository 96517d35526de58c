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
// like the forward solve, in reverse (adjoint_ws.cuh holds the kernel):
// with mu_l = J_l^T lambda_l each step is the affine map
//   mu_l = J_l^T mu_{l+1} + J_l^T g_l,
// whose maps depend only on step l's own data.  Then lambda_l = g_l + mu_{l+1},
// du_l follows from lambda_l by the chain rule of the cell, da sums
// (d pre / d a) du over b and l in a fixed order (deterministic), and the
// gradient of the initial state is mu_1.
//
// This header holds what the scan kernel shares with the host: its
// parameter block and the fixed-order reduction of da.
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

}  // namespace pararnn
