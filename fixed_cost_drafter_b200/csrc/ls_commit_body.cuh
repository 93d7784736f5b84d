// Per-(sequence, layer, KV head, K|V) body of the view extraction from the target's
// verification pass (LongSpark paper page, Figure 2 caption (a)-(b); Figure 3 caption:
// the summary is updated from only the newly retained rows N, Delta = |N| <= B + 1).
// One warp handles one tensor (K or V) of one KV head:
//   1. every load that does not depend on the accept scan is issued first (counters,
//      token ids, all B + 1 verify rows, the fp32 partial / global sums), so the commit
//      costs one memory round trip;
//   2. greedy accept scan (two ballots cover B <= 64 drafts): a, Delta = a + 1;
//   3. rows 0..a go to ring slot (len + i) mod W with 16-byte stores, and the same
//      registers are summed into the rows that close the open segments (i < c) and the
//      rows that open the next ones (i >= c), reduced across the row groups of the warp
//      with shuffles, then folded into the fp32 partial / global sums; a segment whose
//      last row arrived becomes a slot mean (fp32 + the attention's dtype copy). One split
//      row c serves every scale: the scales divide each other and Delta <= s_0, so the
//      only segment boundaries a round can cross all sit at the single multiple of s_0 in
//      (len, len + Delta], i.e. at c = s_0 - len mod s_0.
// Used by the stand-alone commit kernel and by the fused round kernel, so both leave the
// same state.
#pragma once
#include "ls_common.cuh"

namespace ls {

// Outcome of one round for one sequence (identical in every warp that computes it).
struct CommitScan {
  int a;                     // accepted drafts
  int64_t len, newlen;       // retained rows before / after the round
  int64_t nseg[kMaxScales];  // finalised segments per scale before the round
  unsigned closes;           // bit k: scale k finalised a segment this round
};

template <typename T, int ROWS>
__device__ inline void commit_tensor(const Dev& p, int bl, int h, int t, int lane,
                                     const int32_t* __restrict__ draft, const int32_t* __restrict__ target,
                                     const T* __restrict__ vsrc, CommitScan& cs) {
  using E = Elem<T>;
  constexpr int VEC = E::kVec;
  const int b = bl / p.L;
  const int nsc = p.nsc;
  const int64_t* ctr = p.counters + int64_t(bl) * (1 + nsc);
  const int lpr = p.D / VEC;  // lanes per row: a power of two <= 32 (host-checked)
  const int rpi = 32 / lpr;   // rows per warp instruction
  const int c = lane & (lpr - 1), rg = lane / lpr;
  const int cb = c * VEC;
  const int64_t tile = int64_t(bl) * p.Hkv + h;
  const int64_t row_stride = int64_t(p.Hkv) * p.D;

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
  uint4 raw[ROWS];
  const T* src = vsrc + int64_t(bl) * (p.B + 1) * row_stride + int64_t(h) * p.D + cb;
#pragma unroll
  for (int j = 0; j < ROWS; ++j) {
    const int i = rg + j * rpi;
    if (i <= p.B) raw[j] = ld_nc_v4(src + int64_t(i) * row_stride);
  }
  float g[VEC], pr[kMaxScales][VEC];
  float* gp = p.glob + (tile * 2 + t) * p.D + cb;
  if (rg == 0) {
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

  // greedy acceptance: first i with draft[i] != target[i], else B
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

  T* kvt = reinterpret_cast<T*>(p.kv) + (tile * 2 + t) * int64_t(p.R) * p.D;
  float lo[VEC], hi[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) lo[e] = hi[e] = 0.f;
  const int ring0 = int(uint64_t(len) % uint32_t(p.W));
#pragma unroll
  for (int j = 0; j < ROWS; ++j) {
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
    const float inv_len = __frcp_rn(float(newlen));
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
        const float inv_sc = __frcp_rn(float(sc));  // exact for power-of-two scales
#pragma unroll
        for (int e = 0; e < VEC; ++e) m[e] = (pr[k][e] + lo[e]) * inv_sc;
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
      const float inv_cnt = cnt > 0 ? __frcp_rn(float(cnt)) : 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) m[e] = pr[k][e] * inv_cnt;
      *reinterpret_cast<uint4*>(kvt + (row0 + p.slots) * p.D + cb) = E::from_f32(m);
    }
  }
  cs.a = a;
  cs.len = len;
  cs.newlen = newlen;
#pragma unroll
  for (int k = 0; k < kMaxScales; ++k) cs.nseg[k] = nseg[k];
  cs.closes = closes;
}

// The boundary view (Figure 2 caption (b)): the hidden vector at verify row a becomes the
// sequence-layer's boundary state. Each KV head's commit copies its own 1/Hkv slice, so the
// copy is spread over the (sequence, layer)'s commits and costs one round trip: every load
// of a thread is issued before its first store. VEC-element pieces; hidden % VEC == 0.
template <typename T, int kPieces>
__device__ inline void copy_boundary_slice(const Dev& p, int bl, int h, int a, int tid, int nthreads,
                                           const T* __restrict__ vh) {
  constexpr int VEC = Elem<T>::kVec;
  const int pieces = p.hidden / VEC;
  const int per = (pieces + p.Hkv - 1) / p.Hkv;
  const int beg = h * per, end = beg + per < pieces ? beg + per : pieces;
  const T* hrow = vh + (int64_t(bl) * (p.B + 1) + a) * p.hidden;
  T* brow = reinterpret_cast<T*>(p.boundary) + int64_t(bl) * p.hidden;
  for (int x0 = beg + tid; x0 < end; x0 += kPieces * nthreads) {
    uint4 v[kPieces];
#pragma unroll
    for (int u = 0; u < kPieces; ++u)
      if (x0 + u * nthreads < end) v[u] = ld_nc_v4(hrow + int64_t(x0 + u * nthreads) * VEC);
#pragma unroll
    for (int u = 0; u < kPieces; ++u)
      if (x0 + u * nthreads < end) *reinterpret_cast<uint4*>(brow + int64_t(x0 + u * nthreads) * VEC) = v[u];
  }
}

// rows of the verify block a lane may need: ceil((B + 1) / rows per warp instruction)
template <typename T>
__host__ __device__ inline int commit_rows_per_lane(int D, int B) {
  const int lpr = D / Elem<T>::kVec;
  return (B + 1 + (32 / lpr) - 1) / (32 / lpr);
}

}  // namespace ls
