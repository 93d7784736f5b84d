// Device twin of the seeded input generator in synth/__init__.py: the same SplitMix64
// draws (Steele, Lea & Flood 2014, counter-based) and the same Irwin-Hall stand-in for
// N(0,1), written straight into GPU memory. Holds none of the drafting method's
// arithmetic; used only to fill large synthetic inputs for tests and the bench.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t finalise(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t n) {
  return finalise(key + (n + 1) * 0x9E3779B97F4A7C15ull);
}

__device__ __forceinline__ uint16_t bf16_rne(float x) {
  uint32_t u = __float_as_uint(x);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
  return uint16_t(u);
}

// out[((((r*nb + b)*nl + l)*np + p)*nx + x] for the element at (r0+r, b0+b, l0+l, p0+p, x0+x)
__global__ void fill_normal_kernel(void* out, int bf16, uint64_t key, int64_t nb, int64_t nl,
                                   int64_t np, int64_t nx, int64_t total, int64_t r0, int64_t b0,
                                   int64_t l0, int64_t p0, int64_t x0, int head_dim, const float* scale,
                                   int scale_heads, float inv_std) {
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    int64_t t = idx;
    const int64_t x = t % nx; t /= nx;
    const int64_t p = t % np; t /= np;
    const int64_t l = t % nl; t /= nl;
    const int64_t b = t % nb; t /= nb;
    const int64_t r = t;
    const int64_t xg = x0 + x;
    int64_t h, d;
    if (head_dim > 0) { h = xg / head_dim; d = xg - h * head_dim; }
    else { h = xg >> 9; d = xg & 511; }
    const uint64_t ctr = (uint64_t(r0 + r) << 52) | (uint64_t(b0 + b) << 44) |
                         (uint64_t(l0 + l) << 38) | (uint64_t(p0 + p) << 16) |
                         (uint64_t(h) << 9) | uint64_t(d);
    const uint64_t u = draw(key, ctr);
    const int64_t s = int64_t(u & 0xFFFF) + int64_t((u >> 16) & 0xFFFF) +
                      int64_t((u >> 32) & 0xFFFF) + int64_t(u >> 48);
    float z = __fmul_rn(float(s - 131070), inv_std);
    if (scale) z = __fmul_rn(z, scale[(l0 + l) * scale_heads + h]);
    if (bf16) static_cast<uint16_t*>(out)[idx] = bf16_rne(z);
    else static_cast<float*>(out)[idx] = z;
  }
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int lss_fill_normal(void* out, int bf16, uint64_t key, int64_t nr, int64_t nb,
                               int64_t nl, int64_t np, int64_t nx, int64_t r0, int64_t b0,
                               int64_t l0, int64_t p0, int64_t x0, int32_t head_dim, const float* scale,
                               int32_t scale_heads, float inv_std, cudaStream_t stream) {
  const int64_t total = nr * nb * nl * np * nx;
  if (total <= 0) return 0;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (total + 255) / 256;
  const int grid = int(want < int64_t(sms) * 16 ? want : int64_t(sms) * 16);
  fill_normal_kernel<<<grid, 256, 0, stream>>>(out, bf16, key, nb, nl, np, nx, total, r0, b0, l0, p0, x0,
                                               head_dim, scale, scale_heads, inv_std);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}
