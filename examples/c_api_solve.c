/* A plain C host program against the C ABI (include/pararnn.h): a ParaGRU
 * Newton solve on fp32 gates, checked against the library's sequential
 * kernel on the same inputs.  Build (see tests/test_c_example.py):
 *   gcc -std=c99 c_api_solve.c -I include -I $CUDA/include \
 *       -L nonlinear_rnn_newton_b200 -lpararnn -L $CUDA/lib64 -lcudart -lm
 * Exit status 0 when the solve converges and matches within 1e-4. */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime.h>

#include "pararnn.h"

/* deterministic inputs: a linear congruential generator, uniform in [-1, 1) */
static float uniform(unsigned long long* s)
{
    *s = *s * 6364136223846793005ull + 1442695040888963407ull;
    return (float)((*s >> 40) & 0xffffff) / 8388608.0f - 1.0f;
}

#define CHECK(x)                                                             \
    do {                                                                     \
        cudaError_t e_ = (x);                                                \
        if (e_ != cudaSuccess) {                                             \
            fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));         \
            return 2;                                                        \
        }                                                                    \
    } while (0)

int main(void)
{
    const int64_t B = 2, L = 700, D = 136;
    const size_t nu = (size_t)(B * L * 3 * D), na = (size_t)(3 * D), nh = (size_t)(B * L * D);
    float* hu = malloc(nu * sizeof(float));
    float* ha = malloc(na * sizeof(float));
    float* h1 = malloc(nh * sizeof(float));
    float* h2 = malloc(nh * sizeof(float));
    unsigned long long seed = 12345;
    for (size_t i = 0; i < nu; ++i) hu[i] = 2.0f * uniform(&seed);
    for (size_t i = 0; i < na; ++i) ha[i] = 0.5f * uniform(&seed);

    float *du, *da, *dh, *dseq;
    void* ws;
    const size_t wsb = pararnn_gru_workspace_size(B, L, D);
    CHECK(cudaMalloc((void**)&du, nu * sizeof(float)));
    CHECK(cudaMalloc((void**)&da, na * sizeof(float)));
    CHECK(cudaMalloc((void**)&dh, nh * sizeof(float)));
    CHECK(cudaMalloc((void**)&dseq, nh * sizeof(float)));
    CHECK(cudaMalloc(&ws, wsb));
    CHECK(cudaMemcpy(du, hu, nu * sizeof(float), cudaMemcpyHostToDevice));
    CHECK(cudaMemcpy(da, ha, na * sizeof(float), cudaMemcpyHostToDevice));

    int iters = -1;
    float residual = -1.0f;
    pararnn_status st = pararnn_gru_solve(du, PARARNN_F32, da, NULL, dh, B, L, D, 1e-6f, 10, ws, wsb, NULL,
                                          &iters, &residual);
    if (st != PARARNN_OK) {
        fprintf(stderr, "solve: %s (%s)\n", pararnn_status_string(st), pararnn_last_error());
        return 1;
    }
    st = pararnn_gru_sequential(du, PARARNN_F32, da, NULL, dseq, B, L, D, NULL);
    if (st != PARARNN_OK) {
        fprintf(stderr, "sequential: %s\n", pararnn_last_error());
        return 1;
    }
    CHECK(cudaDeviceSynchronize());
    CHECK(cudaMemcpy(h1, dh, nh * sizeof(float), cudaMemcpyDeviceToHost));
    CHECK(cudaMemcpy(h2, dseq, nh * sizeof(float), cudaMemcpyDeviceToHost));
    double err = 0.0;
    for (size_t i = 0; i < nh; ++i) {
        const double e = fabs((double)h1[i] - (double)h2[i]);
        if (e > err || e != e) err = e;
    }
    printf("pararnn %s: iters %d residual %.3e max-abs vs sequential %.3e\n", pararnn_version(), iters,
           (double)residual, err);
    cudaFree(du);
    cudaFree(da);
    cudaFree(dh);
    cudaFree(dseq);
    cudaFree(ws);
    free(hu);
    free(ha);
    free(h1);
    free(h2);
    return err <= 1e-4 ? 0 : 1;
}
