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
// This header holds the scan kernel's parameter block; the fixed-order
// reduction of da is in da_reduce.cuh.
#pragma once

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

}  // namespace pararnn
