/* A plain C99 user of the library on the GPU, with no Python and no PyTorch: the CUDA
 * runtime allocates the buffers, the library runs three fused steps of a small ZeRO-2
 * layout (the first with zero_step, the others with zero_step_device_scalars), and the
 * program writes its inputs and outputs to a file for the test to check against the
 * oracle.  Usage: abi_device_check <output file>. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "zero.h"

#define CHECK(x)                                                       \
    do {                                                               \
        if (!(x)) {                                                    \
            fprintf(stderr, "failed: %s (line %d)\n", #x, __LINE__);  \
            return 1;                                                  \
        }                                                              \
    } while (0)

int main(int argc, char **argv)
{
    if (argc != 2) return 2;
    const int64_t sizes[2] = {70001, 4099};
    const int32_t N = 3;
    zero_layout_desc d = {N, 2, 2, sizes, 7001, 8, 0, NULL, 0};
    zero_layout *L = NULL;
    zero_layout_info info;
    CHECK(zero_layout_create(&d, &L) == ZERO_OK);
    CHECK(zero_layout_get_info(L, &info) == ZERO_OK);
    CHECK(zero_layout_to_device(L, NULL) == ZERO_OK);
    const int64_t P = info.padded, psi = info.psi;

    /* inputs: finite fp16 bit patterns of both signs, zero padding; small fp32 weights */
    uint16_t *g = calloc((size_t)(N * P), sizeof(uint16_t));
    float *master = calloc((size_t)P, sizeof(float));
    uint16_t *p16 = calloc((size_t)P, sizeof(uint16_t));
    float *m = calloc((size_t)P, sizeof(float)), *v = calloc((size_t)P, sizeof(float));
    CHECK(g && master && p16 && m && v);
    for (int32_t r = 0; r < N; ++r)
        for (int64_t i = 0; i < psi; ++i)
            g[r * P + i] = (uint16_t)(0x1800 + (uint16_t)((i * 7 + r * 13) % 0x1400) + (((i + r) & 1) ? 0x8000 : 0));
    for (int64_t i = 0; i < psi; ++i) master[i] = (float)((i % 1000) - 500) * 1e-3f;

    uint16_t *dg, *dp16;
    float *dmaster, *dm, *dv;
    CHECK(cudaMalloc((void **)&dg, (size_t)(N * P) * 2) == cudaSuccess);
    CHECK(cudaMalloc((void **)&dp16, (size_t)P * 2) == cudaSuccess);
    CHECK(cudaMalloc((void **)&dmaster, (size_t)P * 4) == cudaSuccess);
    CHECK(cudaMalloc((void **)&dm, (size_t)P * 4) == cudaSuccess);
    CHECK(cudaMalloc((void **)&dv, (size_t)P * 4) == cudaSuccess);
    CHECK(cudaMemcpy(dg, g, (size_t)(N * P) * 2, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemcpy(dmaster, master, (size_t)P * 4, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemset(dm, 0, (size_t)P * 4) == cudaSuccess);
    CHECK(cudaMemset(dv, 0, (size_t)P * 4) == cudaSuccess);
    CHECK(cudaMemset(dp16, 0, (size_t)P * 2) == cudaSuccess);

    /* step 1 with its scalars passed at launch (zero_step); steps 2 and 3 with the scalars
     * filled on the host and read from device memory (zero_step_device_scalars) */
    zero_step_scalars *dsc;
    CHECK(cudaMalloc((void **)&dsc, sizeof(zero_step_scalars)) == cudaSuccess);
    for (int64_t t = 1; t <= 3; ++t) {
        zero_adamw_hparams hp = {1e-3, 0.9, 0.999, 1e-8, 0.01, 1024.0, t};
        if (t == 1) {
            CHECK(zero_step(L, dg, P, dmaster, dm, dv, NULL, dp16, &hp, NULL, NULL, NULL) == ZERO_OK);
        } else {
            zero_step_scalars sc;
            CHECK(zero_step_scalars_fill(L, &hp, &sc) == ZERO_OK);
            CHECK(cudaMemcpy(dsc, &sc, sizeof sc, cudaMemcpyHostToDevice) == cudaSuccess);
            CHECK(zero_step_device_scalars(L, dg, P, dmaster, dm, dv, NULL, dp16, dsc, NULL, NULL) == ZERO_OK);
        }
    }
    CHECK(zero_get_error(L, NULL) == ZERO_OK);
    cudaFree(dsc);

    float *out_master = malloc((size_t)P * 4), *out_m = malloc((size_t)P * 4), *out_v = malloc((size_t)P * 4);
    CHECK(out_master && out_m && out_v);
    CHECK(cudaMemcpy(out_master, dmaster, (size_t)P * 4, cudaMemcpyDeviceToHost) == cudaSuccess);
    CHECK(cudaMemcpy(out_m, dm, (size_t)P * 4, cudaMemcpyDeviceToHost) == cudaSuccess);
    CHECK(cudaMemcpy(out_v, dv, (size_t)P * 4, cudaMemcpyDeviceToHost) == cudaSuccess);
    CHECK(cudaMemcpy(p16, dp16, (size_t)P * 2, cudaMemcpyDeviceToHost) == cudaSuccess);

    FILE *f = fopen(argv[1], "wb");
    CHECK(f != NULL);
    const int64_t head[2] = {N, P};
    CHECK(fwrite(head, sizeof head, 1, f) == 1);
    CHECK(fwrite(g, 2, (size_t)(N * P), f) == (size_t)(N * P));
    CHECK(fwrite(master, 4, (size_t)P, f) == (size_t)P);
    CHECK(fwrite(out_master, 4, (size_t)P, f) == (size_t)P);
    CHECK(fwrite(out_m, 4, (size_t)P, f) == (size_t)P);
    CHECK(fwrite(out_v, 4, (size_t)P, f) == (size_t)P);
    CHECK(fwrite(p16, 2, (size_t)P, f) == (size_t)P);
    CHECK(fclose(f) == 0);

    cudaFree(dg);
    cudaFree(dp16);
    cudaFree(dmaster);
    cudaFree(dm);
    cudaFree(dv);
    zero_layout_destroy(L);
    printf("ok\n");
    return 0;
}
