// Internal constants and the device-side workspace header shared by the host
// launcher and the kernels.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "pararnn.h"

namespace pararnn {

constexpr int kV = 4;              // channels per lane
constexpr int kDc = 32 * kV;       // channels per tile (one per lane x kV)

// Default limit for every device-side wait (look-back flags, grid barrier,
// TMA completion).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// First 256 bytes of every workspace.  Zeroed by the host before each run.
// Pass boundaries the fused solve timestamps (%globaltimer, ns): the start of
// pass 0 and the end of each of the first kPassTimes - 1 passes.
constexpr int kPassTimes = 16;

struct alignas(256) WsHeader {
    unsigned tick[4];  // tile ticket counter per pass slot (pass k uses k % 3)
    unsigned res[4];   // max |F| bits of the updated states per pass slot
    unsigned res0;     // max |F| bits of the initial guess
    unsigned bar;      // grid barrier arrivals (monotone)
    int error;         // first device-side error (pararnn_status < 0), 0 if none
    int passes;        // Newton passes run
    pararnn_result result;
    unsigned long long t_pass[kPassTimes];  // see kPassTimes (0 = not reached)
    // Segment passes only (the sequence split across GPUs; written by the
    // host after the header is zeroed): the state the first step of chunk 0
    // is linearised at, per component (0 = s0), and whether the first pass
    // starts from the states the state tensor maps point at (1) instead of
    // the zero guess (0).
    unsigned long long seg_lin[2];
    int seg_warm;
    // The pass the fused solve starts with: 0, or 1 when pass 0 ran in the
    // projection kernel (which then left H^1, the residuals of H^0 and H^1
    // in res0 and res[0], and its own ticket count in tick[3]).
    int k0;
    // Per pass slot: a tile of the pass has found a residual above tol (or
    // NaN), so the pass cannot end the solve with its residual reported.
    unsigned over[4];
    unsigned char pad[256 - 4 * 4 * 2 - 4 * 4 - sizeof(pararnn_result) - 8 * kPassTimes - 8 * 2 - 4 - 4 - 4 * 4];
};
static_assert(sizeof(WsHeader) == 256, "workspace header must be 256 bytes");

}  // namespace pararnn
