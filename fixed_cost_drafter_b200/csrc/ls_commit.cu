// View extraction from the target's verification pass: LongSpark paper page,
// Figure 2 caption (a)-(b) and Figure 3 caption (summary updated from only the newly
// retained rows N, Delta = |N| <= B + 1).
//
// One CTA per (sequence, layer). Warp 2h+t owns KV head h, tensor t (0 = K, 1 = V):
//   1. greedy accept scan (every warp, one ballot per 32 drafts): a, Delta = a + 1;
//   2. verify rows 0..a are read once with 16-byte loads (D*e/16 lanes per row, several
//      rows per warp instruction) and written to ring slot (len + i) mod W;
//   3. the same registers are summed into the rows that close the open segments (i < c)
//      and the rows that open the next ones (i >= c), reduced across the row groups of
//      the warp with shuffles, and folded into the fp32 partial / global sums; a segment
//      whose last row arrived becomes a slot mean (fp32 + dtype copy). One split row c
//      serves every scale: the scales divide each other and Delta <= s_0, so the only
//      segment boundaries a round can cross all sit at the single multiple of s_0 in
//      (len, len + Delta], i.e. at c = s_0 - len mod s_0;
//   4. the CTA copies the hidden vector of verify row a into the boundary view.
// Counters are read by every warp before the CTA barrier and written once after it.
#include "ls_common.cuh"

namespace ls {

template <typename T>
__global__ void __launch_bounds__(1024)
commit_round_kernel(Dev p, const int32_t* __restrict__ draft, const int32_t* __restrict__ target,
                    const T* __restrict__ vk, const T* __restrict__ vv,
                    const T* __restrict__ vh, int32_t* __restrict__ accept_len,
                    int32_t* __restrict__ next_token) {
  using E = Elem<T>;
  constexpr int VEC = E::kVec;
  const int bl = blockIdx.x;
  const int b = bl / p.L, l = bl - b * p.L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nsc = p.nsc;
  int64_t* ctr = p.counters + int64_t(bl) * (1 + nsc);

  const int64_t len = ctr[0];
  int64_t nseg[kMaxScales];
#pragma unroll
  for (int k = 0; k < kMaxScales; ++k) nseg[k] = k < nsc ? ctr[1 + k] : 0;

  // (a) greedy acceptance: first i with draft[i] != target[i], else B.
  int a = p.B;
  for (int base = 0; base < p.B; base += 32) {
    const int i = base + lane;
    const bool mism = i < p.B && draft[int64_t(b) * p.B + i] != target[int64_t(b) * (p.B + 1) + i];
    const unsigned m = __ballot_sync(0xffffffffu, mism);
    if (m) { a = base + __ffs(m) - 1; break; }
  }
  const int delta = a + 1;
  const int64_t newlen = len + delta;

  // rows before the split row close the open segments; scale k closes one this round
  // exactly when its own distance to the next boundary is <= Delta (then it equals c)
  const int c_split = int(p.scales[0] - (len - nseg[0] * p.scales[0]));
  unsigned closes = 0;
#pragma unroll
  for (int k = 0; k < kMaxScales; ++k)
    if (k < nsc && p.scales[k] - (len - nseg[k] * p.scales[k]) <= delta) closes |= 1u << k;

  if (warp < 2 * p.Hkv) {
    const int h = warp >> 1, t = warp & 1;
    const int64_t row_stride = int64_t(p.Hkv) * p.D;
    const T* src = (t == 0 ? vk : vv) + int64_t(bl) * (p.B + 1) * row_stride + int64_t(h) * p.D;
    const int64_t tile = int64_t(bl) * p.Hkv + h;
    T* kvt = reinterpret_cast<T*>(p.kv) + (tile * 2 + t) * int64_t(p.R) * p.D;
    const int lpr = p.D / VEC;  // lanes per row: a power of two <= 32 (host-checked)
    const int rpi = 32 / lpr;   // rows per warp instruction
    const int c = lane & (lpr - 1), rg = lane / lpr;

    float lo[VEC], hi[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) lo[e] = hi[e] = 0.f;
    const int ring0 = int(len % p.W);
    for (int i = rg; i < delta; i += rpi) {
      const uint4 raw = ld_nc_v4(src + int64_t(i) * row_stride + c * VEC);
      int slot = ring0 + i;
      if (slot >= p.W) slot -= p.W;  // Delta <= W
      *reinterpret_cast<uint4*>(kvt + int64_t(slot) * p.D + c * VEC) = raw;
      float f[VEC];
      E::to_f32(raw, f);
      if (i < c_split) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) lo[e] += f[e];
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) hi[e] += f[e];
      }
    }
    // segmented reduction across the row groups of the warp
    for (int off = lpr; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        lo[e] += __shfl_xor_sync(0xffffffffu, lo[e], off);
        hi[e] += __shfl_xor_sync(0xffffffffu, hi[e], off);
      }
    }
    if (rg == 0) {
      const int cb = c * VEC;
      // global sum and its mean row
      float* gp = p.glob + (tile * 2 + t) * p.D + cb;
      float g[VEC], m[VEC];
#pragma unroll
      for (int e = 0; e < VEC; e += 4) {
        float4 v4 = *reinterpret_cast<const float4*>(gp + e);
        g[e] = v4.x + (lo[e] + hi[e]); g[e + 1] = v4.y + (lo[e + 1] + hi[e + 1]);
        g[e + 2] = v4.z + (lo[e + 2] + hi[e + 2]); g[e + 3] = v4.w + (lo[e + 3] + hi[e + 3]);
        *reinterpret_cast<float4*>(gp + e) = make_float4(g[e], g[e + 1], g[e + 2], g[e + 3]);
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) m[e] = g[e] / float(newlen);
      *reinterpret_cast<uint4*>(kvt + int64_t(p.R - 1) * p.D + cb) = E::from_f32(m);

#pragma unroll
      for (int k = 0; k < kMaxScales; ++k) {
        if (k >= nsc) break;
        const int s = p.scales[k];
        float* pp = p.part + ((tile * nsc + k) * 2 + t) * p.D + cb;
        float pr[VEC];
#pragma unroll
        for (int e = 0; e < VEC; e += 4) {
          float4 v4 = *reinterpret_cast<const float4*>(pp + e);
          pr[e] = v4.x; pr[e + 1] = v4.y; pr[e + 2] = v4.z; pr[e + 3] = v4.w;
        }
        const bool completes = (closes >> k) & 1u;
        const int64_t row0 = int64_t(p.W) + int64_t(k) * (p.slots + 1);
        if (completes) {
          const int slot = int(nseg[k] % p.slots);
#pragma unroll
          for (int e = 0; e < VEC; ++e) m[e] = (pr[e] + lo[e]) / float(s);
          float* sg = p.seg + (((tile * nsc + k) * p.slots + slot) * 2 + t) * p.D + cb;
#pragma unroll
          for (int e = 0; e < VEC; e += 4)
            *reinterpret_cast<float4*>(sg + e) = make_float4(m[e], m[e + 1], m[e + 2], m[e + 3]);
          *reinterpret_cast<uint4*>(kvt + (row0 + slot) * p.D + cb) = E::from_f32(m);
#pragma unroll
          for (int e = 0; e < VEC; ++e) pr[e] = hi[e];
        } else {  // no boundary crossed at this scale: every row extends the open segment
#pragma unroll
          for (int e = 0; e < VEC; ++e) pr[e] += lo[e] + hi[e];
        }
#pragma unroll
        for (int e = 0; e < VEC; e += 4)
          *reinterpret_cast<float4*>(pp + e) = make_float4(pr[e], pr[e + 1], pr[e + 2], pr[e + 3]);
        const int64_t cnt = newlen - (nseg[k] + (completes ? 1 : 0)) * int64_t(s);
#pragma unroll
        for (int e = 0; e < VEC; ++e) m[e] = cnt > 0 ? pr[e] / float(cnt) : 0.f;
        *reinterpret_cast<uint4*>(kvt + (row0 + p.slots) * p.D + cb) = E::from_f32(m);
      }
    }
  }

  // boundary state: hidden vectors at verify row a
  {
    const T* hrow = vh + (int64_t(bl) * (p.B + 1) + a) * p.hidden;
    T* brow = reinterpret_cast<T*>(p.boundary) + int64_t(bl) * p.hidden;
    for (int x = threadIdx.x * VEC; x < p.hidden; x += blockDim.x * VEC)
      *reinterpret_cast<uint4*>(brow + x) = ld_nc_v4(hrow + x);
  }

  __syncthreads();  // every warp has read the counters
  if (threadIdx.x == 0) {
    ctr[0] = newlen;
    for (int k = 0; k < nsc; ++k) ctr[1 + k] = nseg[k] + ((closes >> k) & 1u);
    if (l == 0) {
      accept_len[b] = a;
      next_token[b] = target[int64_t(b) * (p.B + 1) + a];
    }
  }
}

template __global__ void commit_round_kernel<float>(Dev, const int32_t*, const int32_t*, const float*,
                                                    const float*, const float*, int32_t*, int32_t*);
template __global__ void commit_round_kernel<__nv_bfloat16>(Dev, const int32_t*, const int32_t*,
                                                            const __nv_bfloat16*, const __nv_bfloat16*,
                                                            const __nv_bfloat16*, int32_t*, int32_t*);

cudaError_t launch_commit(const Dev& p, const int32_t* draft, const int32_t* target, const void* vk,
                          const void* vv, const void* vh, int32_t* accept_len, int32_t* next_token,
                          cudaStream_t stream) {
  const int threads = max(64, 64 * p.Hkv);
  const dim3 grid(p.b * p.L);
  if (p.dtype == LS_BF16)
    commit_round_kernel<__nv_bfloat16><<<grid, threads, 0, stream>>>(
        p, draft, target, static_cast<const __nv_bfloat16*>(vk), static_cast<const __nv_bfloat16*>(vv),
        static_cast<const __nv_bfloat16*>(vh), accept_len, next_token);
  else
    commit_round_kernel<float><<<grid, threads, 0, stream>>>(
        p, draft, target, static_cast<const float*>(vk), static_cast<const float*>(vv),
        static_cast<const float*>(vh), accept_len, next_token);
  return cudaGetLastError();
}

}  // namespace ls
