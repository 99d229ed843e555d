// GPU fill of the synthetic counter-based streams (same definition as synth/gen.py):
// splitmix64 output function (Steele, Lea and Flood, OOPSLA 2014) over key + GOLDEN * (c + 1),
// four 16-bit fields summed (Irwin-Hall), centred, one float32 multiply, an optional planted
// float32 shift, then bf16 round-to-nearest-even. Holds no step of the attention method.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint16_t f2bf(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// out[b][j][h][d] for j < n: stream keys[b * H + h], counter (t0[b] + j) * 128 + d.
__global__ void fill_kernel(const uint64_t* __restrict__ keys, int B, int H,
                            const int64_t* __restrict__ t0, int n,
                            const int32_t* __restrict__ n_valid,
                            const int32_t* __restrict__ cl_off, const int32_t* __restrict__ cl_start,
                            const int32_t* __restrict__ cl_len, const float* __restrict__ cl_delta,
                            float inv_std, uint16_t* __restrict__ out) {
  const int j = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  if (n_valid && j >= n_valid[b]) return;
  const int64_t pos = t0[b] + j;
  const uint64_t c = (uint64_t)pos * 128u + (uint64_t)d;
  for (int h = 0; h < H; ++h) {
    const uint64_t w = mix64(keys[b * H + h] + 0x9E3779B97F4A7C15ull * (c + 1u));
    const int s = (int)(w & 0xffffu) + (int)((w >> 16) & 0xffffu) + (int)((w >> 32) & 0xffffu) +
                  (int)(w >> 48) - 2 * 65535;
    float x = __fmul_rn((float)s, inv_std);
    if (cl_off) {
      for (int k = cl_off[b * H + h]; k < cl_off[b * H + h + 1]; ++k) {
        if (pos >= cl_start[k] && pos < cl_start[k] + cl_len[k]) {
          x = __fadd_rn(x, cl_delta[(int64_t)k * 128 + d]);
          break;
        }
      }
    }
    out[(((int64_t)b * n + j) * H + h) * 128 + d] = f2bf(x);
  }
}

}  // namespace

extern "C" int synth_fill_rows(const uint64_t* keys, int B, int H, const int64_t* t0, int n,
                               const int32_t* n_valid, const int32_t* cl_off,
                               const int32_t* cl_start, const int32_t* cl_len,
                               const float* cl_delta, float inv_std, uint16_t* out,
                               cudaStream_t stream) {
  if (!keys || !t0 || !out || B < 1 || H < 1 || n < 0) return -1;
  if (n == 0) return 0;
  fill_kernel<<<dim3(n, B), 128, 0, stream>>>(keys, B, H, t0, n, n_valid, cl_off, cl_start,
                                               cl_len, cl_delta, inv_std, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}
