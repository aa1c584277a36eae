/* A plain C caller of the library (no Python, no torch): allocates two
 * tensors with the CUDA runtime, runs `steps` AdamW steps through the C ABI of
 * include/fp8adam.h and writes the final params, codes, scales and amax to a
 * binary file for comparison with the oracle.
 *
 * usage: c_abi_example <inputs.bin> <outputs.bin> <steps>
 * inputs.bin:  int64 n0, n1; then per tensor: fp32 params[n]; then per step
 *              and tensor: uint16 bf16 gradients[n]
 * outputs.bin: per tensor: fp32 params[n], uint8 m[n], uint8 v[n]; then fp32
 *              scale_m[2], scale_v[2], amax_m[2], amax_v[2]
 * Exit status 0 on success; 2 on bad input; 3 on a CUDA or library error. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime_api.h>

#include "fp8adam.h"

#define CHECK_CUDA(x) \
  do {                \
    if ((x) != cudaSuccess) return 3; \
  } while (0)
#define CHECK_LIB(x)  \
  do {                \
    int rc_ = (x);    \
    if (rc_ != FP8ADAM_OK) { fprintf(stderr, "%s\n", fp8adam_strerror(rc_)); return 3; } \
  } while (0)

static int read_all(FILE* f, void* dst, size_t bytes) { return fread(dst, 1, bytes, f) == bytes ? 0 : 2; }

int main(int argc, char** argv) {
  if (argc != 4) return 2;
  const int steps = atoi(argv[3]);
  FILE* in = fopen(argv[1], "rb");
  if (!in || steps < 1) return 2;
  int64_t n[2];
  if (read_all(in, n, sizeof(n))) return 2;
  if (n[0] <= 0 || n[1] <= 0 || n[0] > (1 << 26) || n[1] > (1 << 26)) return 2;

  float* p_dev[2];
  uint16_t* g_dev[2];
  uint8_t *m_dev[2], *v_dev[2];
  float* state_dev; /* scale_m[2], scale_v[2], amax_m[2], amax_v[2] */
  fp8adam_tensor t[2];
  for (int i = 0; i < 2; ++i) {
    float* p_host = (float*)malloc((size_t)n[i] * sizeof(float));
    if (!p_host || read_all(in, p_host, (size_t)n[i] * sizeof(float))) return 2;
    CHECK_CUDA(cudaMalloc((void**)&p_dev[i], (size_t)n[i] * sizeof(float)));
    CHECK_CUDA(cudaMalloc((void**)&g_dev[i], (size_t)n[i] * sizeof(uint16_t)));
    CHECK_CUDA(cudaMalloc((void**)&m_dev[i], (size_t)n[i]));
    CHECK_CUDA(cudaMalloc((void**)&v_dev[i], (size_t)n[i]));
    CHECK_CUDA(cudaMemcpy(p_dev[i], p_host, (size_t)n[i] * sizeof(float), cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemset(m_dev[i], 0, (size_t)n[i]));
    CHECK_CUDA(cudaMemset(v_dev[i], 0, (size_t)n[i]));
    free(p_host);
    t[i].param = p_dev[i];
    t[i].grad = g_dev[i];
    t[i].m = m_dev[i];
    t[i].v = v_dev[i];
    t[i].numel = n[i];
  }
  const float init[8] = {1.0f, 1.0f, 1.0f, 1.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  CHECK_CUDA(cudaMalloc((void**)&state_dev, sizeof(init)));
  CHECK_CUDA(cudaMemcpy(state_dev, init, sizeof(init), cudaMemcpyHostToDevice));

  fp8adam_ctx* ctx = NULL;
  CHECK_LIB(fp8adam_create(t, 2, state_dev, state_dev + 2, state_dev + 4, state_dev + 6, FP8ADAM_E4M3,
                           FP8ADAM_E5M2, 0u, &ctx));
  for (int k = 1; k <= steps; ++k) {
    for (int i = 0; i < 2; ++i) {
      uint16_t* g_host = (uint16_t*)malloc((size_t)n[i] * sizeof(uint16_t));
      if (!g_host || read_all(in, g_host, (size_t)n[i] * sizeof(uint16_t))) return 2;
      CHECK_CUDA(cudaMemcpy(g_dev[i], g_host, (size_t)n[i] * sizeof(uint16_t), cudaMemcpyHostToDevice));
      free(g_host);
    }
    CHECK_LIB(fp8adam_step(ctx, 3e-4f, 0.9f, 0.95f, 1e-8f, 0.1f, (int64_t)k, NULL));
  }
  CHECK_LIB(fp8adam_check(ctx, NULL));
  CHECK_CUDA(cudaDeviceSynchronize());
  fclose(in);

  FILE* out = fopen(argv[2], "wb");
  if (!out) return 2;
  for (int i = 0; i < 2; ++i) {
    void* buf = malloc((size_t)n[i] * sizeof(float));
    if (!buf) return 2;
    CHECK_CUDA(cudaMemcpy(buf, p_dev[i], (size_t)n[i] * sizeof(float), cudaMemcpyDeviceToHost));
    fwrite(buf, sizeof(float), (size_t)n[i], out);
    CHECK_CUDA(cudaMemcpy(buf, m_dev[i], (size_t)n[i], cudaMemcpyDeviceToHost));
    fwrite(buf, 1, (size_t)n[i], out);
    CHECK_CUDA(cudaMemcpy(buf, v_dev[i], (size_t)n[i], cudaMemcpyDeviceToHost));
    fwrite(buf, 1, (size_t)n[i], out);
    free(buf);
  }
  float state[8];
  CHECK_CUDA(cudaMemcpy(state, state_dev, sizeof(state), cudaMemcpyDeviceToHost));
  fwrite(state, sizeof(float), 8, out);
  fclose(out);
  CHECK_LIB(fp8adam_destroy(ctx));
  for (int i = 0; i < 2; ++i) {
    cudaFree(p_dev[i]);
    cudaFree(g_dev[i]);
    cudaFree(m_dev[i]);
    cudaFree(v_dev[i]);
  }
  cudaFree(state_dev);
  return 0;
}
