// View extraction from the target's verification pass: LongSpark paper page,
// Figure 2 caption (a)-(b) and Figure 3 caption (summary updated from only the newly
// retained rows N, Delta = |N| <= B + 1).
//
// One CTA of two warps per (sequence, layer, KV head); warp t owns tensor t (0 = K,
// 1 = V) of that head:
//   1. greedy accept scan (two ballots cover B <= 64 drafts): a, Delta = a + 1;
//   2. every load that does not depend on the scan is issued first (counters, token ids,
//      all B + 1 verify rows, the fp32 partial / global sums), so the commit costs one
//      memory round trip; rows 0..a go to ring slot (len + i) mod W with 16-byte stores;
//   3. the same registers are summed into the rows that close the open segments (i < c)
//      and the rows that open the next ones (i >= c), reduced across the row groups of
//      the warp with shuffles, and folded into the fp32 partial / global sums; a segment
//      whose last row arrived becomes a slot mean (fp32 + dtype copy). One split row c
//      serves every scale: the scales divide each other and Delta <= s_0, so the only
//      segment boundaries a round can cross all sit at the single multiple of s_0 in
//      (len, len + Delta], i.e. at c = s_0 - len mod s_0;
//   4. the head-0 CTA of a (sequence, layer) copies verify row a's hidden vectors into
//      the boundary view;
//   5. the last of the (sequence, layer)'s KV-head CTAs to finish (an arrival counter)
//      writes the new counters, after every CTA has read the old ones.
#include "ls_common.cuh"

namespace ls {

template <typename T, int ROWS>
__global__ void __launch_bounds__(64)
commit_round_kernel(Dev p, const int32_t* __restrict__ draft, const int32_t* __restrict__ target,
                    const T* __restrict__ vk, const T* __restrict__ vv,
                    const T* __restrict__ vh, int32_t* __restrict__ accept_len,
                    int32_t* __restrict__ next_token) {
  using E = Elem<T>;
  constexpr int VEC = E::kVec;
  constexpr int kMaxRowsPerLane = ROWS;  // >= ceil((B + 1) / rows per warp instruction)
  const int bl = blockIdx.x / p.Hkv, h = blockIdx.x - bl * p.Hkv;
  const int b = bl / p.L, l = bl - b * p.L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nsc = p.nsc;
  int64_t* ctr = p.counters + int64_t(bl) * (1 + nsc);
  const bool mover = true;
  const int t = warp;
  const int lpr = p.D / VEC;  // lanes per row: a power of two <= 32 (host-checked)
  const int rpi = 32 / lpr;   // rows per warp instruction
  const int c = lane & (lpr - 1), rg = lane / lpr;
  const int cb = c * VEC;
  const int64_t tile = int64_t(bl) * p.Hkv + h;
  const int64_t row_stride = int64_t(p.Hkv) * p.D;

  // Every load that does not depend on the accept scan is issued first, so the round
  // costs one memory round trip: counters, token ids, all B + 1 verify rows of this
  // warp's (head, K|V) and the fp32 partial / global sums it will update.
  const int64_t len = ctr[0];
  int64_t nseg[kMaxScales];
#pragma unroll
  for (int k = 0; k < kMaxScales; ++k) nseg[k] = k < nsc ? ctr[1 + k] : 0;
  bool mism[2];
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const int i = 32 * w + lane;
    mism[w] = i < p.B && draft[int64_t(b) * p.B + i] != target[int64_t(b) * (p.B + 1) + i];
  }
  uint4 raw[kMaxRowsPerLane];
  const T* src = (t == 0 ? vk : vv) + int64_t(bl) * (p.B + 1) * row_stride + int64_t(h) * p.D + cb;
  if (mover) {
#pragma unroll
    for (int j = 0; j < kMaxRowsPerLane; ++j) {
      const int i = rg + j * rpi;
      if (i <= p.B) raw[j] = ld_nc_v4(src + int64_t(i) * row_stride);
    }
  }
  float g[VEC], pr[kMaxScales][VEC];
  float* gp = p.glob + (tile * 2 + t) * p.D + cb;
  if (mover && rg == 0) {
#pragma unroll
    for (int e = 0; e < VEC; e += 4) {
      const float4 v4 = *reinterpret_cast<const float4*>(gp + e);
      g[e] = v4.x; g[e + 1] = v4.y; g[e + 2] = v4.z; g[e + 3] = v4.w;
    }
#pragma unroll
    for (int k = 0; k < kMaxScales; ++k) {
      if (k < nsc) {
        const float* pp = p.part + ((tile * nsc + k) * 2 + t) * p.D + cb;
#pragma unroll
        for (int e = 0; e < VEC; e += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(pp + e);
          pr[k][e] = v4.x; pr[k][e + 1] = v4.y; pr[k][e + 2] = v4.z; pr[k][e + 3] = v4.w;
        }
      }
    }
  }

  // (a) greedy acceptance: first i with draft[i] != target[i], else B.
  const unsigned m0 = __ballot_sync(0xffffffffu, mism[0]);
  const unsigned m1 = __ballot_sync(0xffffffffu, mism[1]);
  const int a = m0 ? __ffs(m0) - 1 : (m1 ? 32 + __ffs(m1) - 1 : p.B);
  const int delta = a + 1;
  const int64_t newlen = len + delta;

  // rows before the split row close the open segments; scale k closes one this round
  // exactly when its own distance to the next boundary is <= Delta (then it equals c)
  const int c_split = int(p.scales[0] - (len - nseg[0] * p.scales[0]));
  unsigned closes = 0;
#pragma unroll
  for (int k = 0; k < kMaxScales; ++k)
    if (k < nsc && p.scales[k] - (len - nseg[k] * p.scales[k]) <= delta) closes |= 1u << k;

  if (mover) {
    T* kvt = reinterpret_cast<T*>(p.kv) + (tile * 2 + t) * int64_t(p.R) * p.D;
    float lo[VEC], hi[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) lo[e] = hi[e] = 0.f;
    const int ring0 = int(uint64_t(len) % uint32_t(p.W));
#pragma unroll
    for (int j = 0; j < kMaxRowsPerLane; ++j) {
      const int i = rg + j * rpi;
      if (i < delta) {
        int slot = ring0 + i;
        if (slot >= p.W) slot -= p.W;  // Delta <= W
        *reinterpret_cast<uint4*>(kvt + int64_t(slot) * p.D + cb) = raw[j];
        float f[VEC];
        E::to_f32(raw[j], f);
        if (i < c_split) {
#pragma unroll
          for (int e = 0; e < VEC; ++e) lo[e] += f[e];
        } else {
#pragma unroll
          for (int e = 0; e < VEC; ++e) hi[e] += f[e];
        }
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
      float m[VEC];
      // global sum and its mean row
#pragma unroll
      for (int e = 0; e < VEC; ++e) g[e] += lo[e] + hi[e];
#pragma unroll
      for (int e = 0; e < VEC; e += 4)
        *reinterpret_cast<float4*>(gp + e) = make_float4(g[e], g[e + 1], g[e + 2], g[e + 3]);
      // mean rows are the attention's copy: one reciprocal per count, then multiplies
      const float inv_len = 1.0f / float(newlen);
#pragma unroll
      for (int e = 0; e < VEC; ++e) m[e] = g[e] * inv_len;
      *reinterpret_cast<uint4*>(kvt + int64_t(p.R - 1) * p.D + cb) = E::from_f32(m);

#pragma unroll
      for (int k = 0; k < kMaxScales; ++k) {
        if (k >= nsc) break;
        const int sc = p.scales[k];
        float* pp = p.part + ((tile * nsc + k) * 2 + t) * p.D + cb;
        const bool completes = (closes >> k) & 1u;
        const int64_t row0 = int64_t(p.W) + int64_t(k) * (p.slots + 1);
        if (completes) {
          const int slot = int(uint64_t(nseg[k]) % uint32_t(p.slots));
#pragma unroll
          for (int e = 0; e < VEC; ++e) m[e] = (pr[k][e] + lo[e]) / float(sc);
          float* sg = p.seg + (((tile * nsc + k) * p.slots + slot) * 2 + t) * p.D + cb;
#pragma unroll
          for (int e = 0; e < VEC; e += 4)
            *reinterpret_cast<float4*>(sg + e) = make_float4(m[e], m[e + 1], m[e + 2], m[e + 3]);
          *reinterpret_cast<uint4*>(kvt + (row0 + slot) * p.D + cb) = E::from_f32(m);
#pragma unroll
          for (int e = 0; e < VEC; ++e) pr[k][e] = hi[e];
        } else {  // no boundary crossed at this scale: every row extends the open segment
#pragma unroll
          for (int e = 0; e < VEC; ++e) pr[k][e] += lo[e] + hi[e];
        }
#pragma unroll
        for (int e = 0; e < VEC; e += 4)
          *reinterpret_cast<float4*>(pp + e) = make_float4(pr[k][e], pr[k][e + 1], pr[k][e + 2], pr[k][e + 3]);
        const int64_t cnt = newlen - (nseg[k] + (completes ? 1 : 0)) * int64_t(sc);
        const float inv_cnt = cnt > 0 ? 1.0f / float(cnt) : 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) m[e] = pr[k][e] * inv_cnt;
        *reinterpret_cast<uint4*>(kvt + (row0 + p.slots) * p.D + cb) = E::from_f32(m);
      }
    }
  }

  // boundary state: hidden vectors at verify row a
  if (h == 0) {
    const T* hrow = vh + (int64_t(bl) * (p.B + 1) + a) * p.hidden;
    T* brow = reinterpret_cast<T*>(p.boundary) + int64_t(bl) * p.hidden;
    for (int x = threadIdx.x * VEC; x < p.hidden; x += blockDim.x * VEC)
      *reinterpret_cast<uint4*>(brow + x) = ld_nc_v4(hrow + x);
  }

  __syncthreads();  // both warps have read the counters
  if (threadIdx.x == 0) {
    // the last KV-head CTA of this (sequence, layer) to arrive writes the new counters:
    // every other one has read the old counters before its own arrival
    const int before = atomicAdd(p.arrive + bl, 1);
    if (before == p.Hkv - 1) {
      p.arrive[bl] = 0;
      ctr[0] = newlen;
      for (int k = 0; k < nsc; ++k) ctr[1 + k] = nseg[k] + ((closes >> k) & 1u);
      if (l == 0) {
        accept_len[b] = a;
        next_token[b] = target[int64_t(b) * (p.B + 1) + a];
      }
    }
  }
}

template <typename T, int ROWS>
static void launch_commit_t(const Dev& p, const int32_t* draft, const int32_t* target, const void* vk,
                            const void* vv, const void* vh, int32_t* accept_len, int32_t* next_token,
                            cudaStream_t stream) {
  commit_round_kernel<T, ROWS><<<p.b * p.L * p.Hkv, 64, 0, stream>>>(
      p, draft, target, static_cast<const T*>(vk), static_cast<const T*>(vv), static_cast<const T*>(vh),
      accept_len, next_token);
}

template <typename T>
static void launch_commit_dt(const Dev& p, const int32_t* draft, const int32_t* target, const void* vk,
                             const void* vv, const void* vh, int32_t* accept_len, int32_t* next_token,
                             cudaStream_t stream) {
  const int lpr = p.D / Elem<T>::kVec;
  const int rows = (p.B + 1 + (32 / lpr) - 1) / (32 / lpr);
  if (rows <= 9) launch_commit_t<T, 9>(p, draft, target, vk, vv, vh, accept_len, next_token, stream);
  else if (rows <= 17) launch_commit_t<T, 17>(p, draft, target, vk, vv, vh, accept_len, next_token, stream);
  else launch_commit_t<T, 33>(p, draft, target, vk, vv, vh, accept_len, next_token, stream);
}

cudaError_t launch_commit(const Dev& p, const int32_t* draft, const int32_t* target, const void* vk,
                          const void* vv, const void* vh, int32_t* accept_len, int32_t* next_token,
                          cudaStream_t stream) {
  if (p.dtype == LS_BF16)
    launch_commit_dt<__nv_bfloat16>(p, draft, target, vk, vv, vh, accept_len, next_token, stream);
  else
    launch_commit_dt<float>(p, draft, target, vk, vv, vh, accept_len, next_token, stream);
  return cudaGetLastError();
}

}  // namespace ls
