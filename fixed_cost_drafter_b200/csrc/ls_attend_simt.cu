// Drafter block attention over the three views on CUDA cores: LongSpark paper page,
// Figure 2 caption (c). Used for fp32 states and for shapes the tcgen05 kernel does
// not tile (GQA group x block != 64, head_dim != 128, or too many view rows).
//
// One CTA (8 warps) per (KV head g, layer, sequence). The M = (Hq/Hkv) * B query rows
// of the group sit in shared memory as fp32; keys/values stream through shared memory
// 32 slots at a time (slot 0 = boundary, slot 1 + r = arena row r of the tile); each
// warp keeps an online softmax (running max, running sum, output in registers) for
// its query rows, one key per lane for the logits and D/32 output columns per lane.
// `views` (LS_VIEW_*) selects the views that take part (Table 5's component ablations);
// a row with no valid slot at all writes zeros.
#include "ls_common.cuh"

namespace ls {

constexpr int kSimtWarps = 8;
constexpr int kSimtRowsPerWarp = 8;  // M <= 64

template <typename T, int DV>
__global__ void __launch_bounds__(kSimtWarps * 32)
attend_simt_kernel(Dev p, int layer_begin, int layer_count, const T* __restrict__ q,
                   const T* __restrict__ bk, const T* __restrict__ bv, int64_t bstride,
                   float scale, int views, void* __restrict__ out) {
  using E = Elem<T>;
  const int g = blockIdx.x, lc = blockIdx.y, b = blockIdx.z;
  const int l = layer_begin + lc;
  const int D = DV * 32;
  const int grp = p.Hq / p.Hkv;
  const int M = grp * p.B;
  const int S = 1 + p.R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  extern __shared__ float sm[];
  float* qs = sm;                       // [M][D]
  float* ks = qs + M * D;               // [32][D + 1]
  float* vs = ks + 32 * (D + 1);        // [32][D]
  __shared__ int valid_s[32];

  const int64_t* ctr = p.counters + (int64_t(b) * p.L + l) * (1 + p.nsc);
  const int64_t len = ctr[0];
  int64_t nseg[kMaxScales];
#pragma unroll
  for (int k = 0; k < kMaxScales; ++k) nseg[k] = k < p.nsc ? ctr[1 + k] : 0;

  // query rows m = i * grp + j  <->  q[b][lc][i][g*grp + j][:]
  for (int x = threadIdx.x; x < M * D; x += blockDim.x) {
    const int m = x / D, d = x - m * D;
    const int i = m / grp, j = m - i * grp;
    qs[x] = E::load1(q, (((int64_t(b) * layer_count + lc) * p.B + i) * p.Hq + g * grp + j) * D + d);
  }

  const int64_t tile = (int64_t(b) * p.L + l) * p.Hkv + g;
  const T* kbase = reinterpret_cast<const T*>(p.kv) + tile * 2 * int64_t(p.R) * D;
  const T* vbase = kbase + int64_t(p.R) * D;
  const int64_t boff = (int64_t(b) * p.L + l) * bstride + int64_t(g) * D;

  float mrun[kSimtRowsPerWarp], lrun[kSimtRowsPerWarp], o[kSimtRowsPerWarp][DV];
#pragma unroll
  for (int r = 0; r < kSimtRowsPerWarp; ++r) {
    mrun[r] = -INFINITY; lrun[r] = 0.f;
#pragma unroll
    for (int dd = 0; dd < DV; ++dd) o[r][dd] = 0.f;
  }

  for (int s0 = 0; s0 < S; s0 += 32) {
    __syncthreads();
    for (int x = threadIdx.x; x < 32 * D; x += blockDim.x) {
      const int j = x / D, d = x - j * D;
      const int s = s0 + j;
      float kx = 0.f, vx = 0.f;
      if (s == 0) {
        kx = E::load1(bk, boff + d); vx = E::load1(bv, boff + d);
      } else if (s < S) {
        kx = E::load1(kbase, int64_t(s - 1) * D + d); vx = E::load1(vbase, int64_t(s - 1) * D + d);
      }
      ks[j * (D + 1) + d] = kx;
      vs[j * D + d] = vx;
    }
    if (threadIdx.x < 32) {
      const int s = s0 + threadIdx.x;
      bool ok = false;
      if (s == 0) ok = (views & LS_VIEW_BOUNDARY) != 0;
      else if (s < S) ok = ((views & (s - 1 < p.W ? LS_VIEW_WINDOW : LS_VIEW_SUMMARY)) != 0) &&
                           arena_row_valid(p, s - 1, len, nseg);
      valid_s[threadIdx.x] = int(ok);
    }
    __syncthreads();
    const bool ok = valid_s[lane] != 0;
#pragma unroll
    for (int r = 0; r < kSimtRowsPerWarp; ++r) {
      const int m = warp + r * kSimtWarps;
      if (m >= M) break;
      const float* qr = qs + m * D;
      float lg = 0.f;
      for (int d = 0; d < D; ++d) lg = fmaf(qr[d], ks[lane * (D + 1) + d], lg);
      lg = ok ? lg * scale : -INFINITY;
      float cmax = lg;
      for (int off = 16; off; off >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, off));
      const float mnew = fmaxf(mrun[r], cmax);
      if (mnew == -INFINITY) continue;  // nothing valid yet in this row
      const float alpha = __expf(mrun[r] - mnew);
      const float pj = ok ? __expf(lg - mnew) : 0.f;
      float psum = pj;
      for (int off = 16; off; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
      lrun[r] = lrun[r] * alpha + psum;
      mrun[r] = mnew;
#pragma unroll
      for (int dd = 0; dd < DV; ++dd) o[r][dd] *= alpha;
      for (int j = 0; j < 32; ++j) {
        const float pb = __shfl_sync(0xffffffffu, pj, j);
#pragma unroll
        for (int dd = 0; dd < DV; ++dd) o[r][dd] = fmaf(pb, vs[j * D + lane + 32 * dd], o[r][dd]);
      }
    }
  }

#pragma unroll
  for (int r = 0; r < kSimtRowsPerWarp; ++r) {
    const int m = warp + r * kSimtWarps;
    if (m >= M) break;
    const int i = m / grp, j = m - i * grp;
    const float inv = lrun[r] > 0.f ? 1.0f / lrun[r] : 0.f;  // no valid slot: zeros
    const int64_t ob = (((int64_t(b) * layer_count + lc) * p.B + i) * p.Hq + g * grp + j) * D;
#pragma unroll
    for (int dd = 0; dd < DV; ++dd) {
      if (p.out_f32) static_cast<float*>(out)[ob + lane + 32 * dd] = o[r][dd] * inv;
      else E::store1(out, ob + lane + 32 * dd, o[r][dd] * inv);
    }
  }
}

template <typename T, int DV>
static cudaError_t launch_simt_t(const Dev& p, int lb, int lcount, const void* q, const void* bk,
                                 const void* bv, int64_t bstride, float scale, int views, void* out,
                                 cudaStream_t stream) {
  const int D = DV * 32;
  const int M = (p.Hq / p.Hkv) * p.B;
  const size_t smem = size_t(M * D + 32 * (D + 1) + 32 * D) * sizeof(float);
  auto kern = attend_simt_kernel<T, DV>;
  // per launch: the opt-in belongs to the current device's copy of the kernel
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(p.Hkv, lcount, p.b);
  kern<<<grid, kSimtWarps * 32, smem, stream>>>(p, lb, lcount, static_cast<const T*>(q),
                                                static_cast<const T*>(bk), static_cast<const T*>(bv),
                                                bstride, scale, views, out);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_simt_dt(const Dev& p, int lb, int lcount, const void* q, const void* bk,
                                  const void* bv, int64_t bstride, float scale, int views, void* out,
                                  cudaStream_t stream) {
  switch (p.D / 32) {
    case 1: return launch_simt_t<T, 1>(p, lb, lcount, q, bk, bv, bstride, scale, views, out, stream);
    case 2: return launch_simt_t<T, 2>(p, lb, lcount, q, bk, bv, bstride, scale, views, out, stream);
    case 4: return launch_simt_t<T, 4>(p, lb, lcount, q, bk, bv, bstride, scale, views, out, stream);
    case 8: return launch_simt_t<T, 8>(p, lb, lcount, q, bk, bv, bstride, scale, views, out, stream);
    default: return cudaErrorInvalidValue;
  }
}

bool simt_supported(const Dev& p) {
  const int M = (p.Hq / p.Hkv) * p.B;
  const int dv = p.D / 32;
  return p.D % 32 == 0 && (dv == 1 || dv == 2 || dv == 4 || dv == 8) &&
         M <= kSimtWarps * kSimtRowsPerWarp;
}

cudaError_t launch_attend_simt(const Dev& p, int lb, int lcount, const void* q, const void* bk,
                               const void* bv, int64_t bstride, float scale, int views, void* out,
                               cudaStream_t stream) {
  if (p.dtype == LS_BF16)
    return launch_simt_dt<__nv_bfloat16>(p, lb, lcount, q, bk, bv, bstride, scale, views, out, stream);
  return launch_simt_dt<float>(p, lb, lcount, q, bk, bv, bstride, scale, views, out, stream);
}

}  // namespace ls
