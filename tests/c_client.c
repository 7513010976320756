/*
 * c_client.c -- a plain C program that drives libadamw4 through its C ABI
 * only (include/adamw4.h), with the CUDA runtime for device memory.  Used by
 * tests/test_c_client.py: it reads a tensor list, weights and per-step
 * gradients from a file, runs the steps, and writes the weights and the
 * exported state blob back, for the test to compare with the oracle.
 *
 * Input file (little-endian):
 *   int32 n, int32 steps, int32 vcode, int32 pad, uint64 seed, int64 total_steps
 *   per tensor: int64 numel, uint32 tensor_id, uint32 flags, float weight_decay, int32 pad
 *   per tensor: numel fp32 weights
 *   per step, per tensor: numel bf16 gradient bit patterns
 * Output file: per tensor numel fp32 weights, then int64 blob length and the blob.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "adamw4.h"

#define CHECK(cond, ...)                  \
    do {                                  \
        if (!(cond)) {                    \
            fprintf(stderr, __VA_ARGS__); \
            fprintf(stderr, "\n");        \
            return 1;                     \
        }                                 \
    } while (0)

static int read_all(FILE *f, void *p, size_t n) { return fread(p, 1, n, f) == n; }

int main(int argc, char **argv)
{
    CHECK(argc == 3, "usage: c_client <input> <output>");
    FILE *in = fopen(argv[1], "rb");
    CHECK(in != NULL, "cannot open %s", argv[1]);
    int32_t head[4];
    uint64_t seed;
    int64_t total_steps;
    CHECK(read_all(in, head, sizeof head) && read_all(in, &seed, 8) && read_all(in, &total_steps, 8),
          "short header");
    const int n = head[0], steps = head[1], vcode = head[2];
    CHECK(n > 0 && n <= 64 && steps > 0, "bad header");

    adamw4_tensor desc[64];
    float *d_w[64];
    uint16_t *d_g[64];
    float *h_w[64];
    uint16_t *h_g[64];
    for (int i = 0; i < n; ++i) {
        int64_t numel;
        uint32_t id, flags;
        float wd;
        int32_t pad;
        CHECK(read_all(in, &numel, 8) && read_all(in, &id, 4) && read_all(in, &flags, 4) &&
                  read_all(in, &wd, 4) && read_all(in, &pad, 4),
              "short tensor record");
        CHECK(cudaMalloc((void **)&d_w[i], (size_t)numel * 4) == cudaSuccess, "cudaMalloc");
        CHECK(cudaMalloc((void **)&d_g[i], (size_t)numel * 2) == cudaSuccess, "cudaMalloc");
        h_w[i] = (float *)malloc((size_t)numel * 4);
        h_g[i] = (uint16_t *)malloc((size_t)numel * 2);
        CHECK(h_w[i] != NULL && h_g[i] != NULL, "malloc");
        desc[i].param = d_w[i];
        desc[i].grad_bf16 = d_g[i];
        desc[i].numel = numel;
        desc[i].tensor_id = id;
        desc[i].flags = flags;
        desc[i].weight_decay = wd;
        desc[i].elem_offset = 0;
    }
    for (int i = 0; i < n; ++i) {
        CHECK(read_all(in, h_w[i], (size_t)desc[i].numel * 4), "short weights");
        CHECK(cudaMemcpy(d_w[i], h_w[i], (size_t)desc[i].numel * 4, cudaMemcpyHostToDevice) ==
                  cudaSuccess,
              "cudaMemcpy");
    }

    adamw4_config cfg = {1e-3f, 0.9f, 0.999f, 1e-8f, vcode, seed, total_steps};
    adamw4_handle *h = NULL;
    int rc = adamw4_create(&cfg, desc, n, 0, &h);
    CHECK(rc == ADAMW4_OK, "adamw4_create: %d %s", rc, adamw4_last_error(NULL));

    for (int s = 0; s < steps; ++s) {
        for (int i = 0; i < n; ++i) {
            CHECK(read_all(in, h_g[i], (size_t)desc[i].numel * 2), "short grads");
            CHECK(cudaMemcpy(d_g[i], h_g[i], (size_t)desc[i].numel * 2, cudaMemcpyHostToDevice) ==
                      cudaSuccess,
                  "cudaMemcpy");
        }
        rc = adamw4_step(h, 1e-3f, NULL);
        CHECK(rc == ADAMW4_OK, "adamw4_step: %d %s", rc, adamw4_last_error(h));
        rc = adamw4_sync(h, NULL);
        CHECK(rc == ADAMW4_OK, "adamw4_sync: %d %s", rc, adamw4_last_error(h));
    }
    fclose(in);

    int64_t t = -1, used = 0;
    CHECK(adamw4_get_step(h, &t) == ADAMW4_OK && t == steps, "step counter");
    CHECK(adamw4_state_export(h, NULL, 0, &used) == ADAMW4_OK && used > 40, "export size query");
    void *blob = malloc((size_t)used);
    CHECK(blob != NULL, "malloc");
    int64_t used2 = 0;
    CHECK(adamw4_state_export(h, blob, used - 1, &used2) == ADAMW4_ERANGE && used2 == used,
          "a buffer one byte short must be refused");
    CHECK(adamw4_state_export(h, blob, used, &used) == ADAMW4_OK, "export");

    FILE *out = fopen(argv[2], "wb");
    CHECK(out != NULL, "cannot open %s", argv[2]);
    for (int i = 0; i < n; ++i) {
        CHECK(cudaMemcpy(h_w[i], d_w[i], (size_t)desc[i].numel * 4, cudaMemcpyDeviceToHost) ==
                  cudaSuccess,
              "cudaMemcpy");
        fwrite(h_w[i], 4, (size_t)desc[i].numel, out);
    }
    fwrite(&used, 8, 1, out);
    fwrite(blob, 1, (size_t)used, out);
    fclose(out);

    CHECK(adamw4_destroy(h) == ADAMW4_OK, "destroy");
    CHECK(adamw4_destroy(h) == ADAMW4_EINVAL, "double destroy must be refused");
    for (int i = 0; i < n; ++i) {
        cudaFree(d_w[i]);
        cudaFree(d_g[i]);
        free(h_w[i]);
        free(h_g[i]);
    }
    free(blob);
    printf("ok\n");
    return 0;
}
