// Per-(sequence, layer, KV head, K|V) body of the view extraction from the target's
// verification pass (LongSpark paper page, Figure 2 caption (a)-(b); Figure 3 caption:
// the summary is updated from only the newly retained rows N, Delta = |N| <= B + 1).
// One warp handles one tensor (K or V) of one KV head, in two phases:
//   load_scan  the counters and token ids first, then the greedy accept scan (two
//              ballots cover B <= 64 drafts): a, Delta = a + 1. Only then are the bulk
//              inputs issued (the retained verify rows 0..a, from the dense verify block
//              or the target's paged cache, and the fp32 partial / global sums), so
//              the few scan inputs do not queue behind them and the loads that need a
//              (the boundary slice) join the same round trip.
//   apply      rows 0..a go to ring slot (len + i) mod W with 16-byte stores, and the same
//              registers are summed into the rows that close the open segments (i < c) and
//              the rows that open the next ones (i >= c), reduced across the row groups of
//              the warp with shuffles, then folded into the fp32 partial / global sums; a
//              segment whose last row arrived becomes a slot mean (fp32 + the attention's
//              dtype copy). One split row c serves every scale: the scales divide each
//              other and Delta <= s_0, so the only segment boundaries a round can cross all
//              sit at the single multiple of s_0 in (len, len + Delta], i.e. at
//              c = s_0 - len mod s_0.
// Between the phases the caller can issue work that needs a (the boundary slice's loads,
// the arrival counter), so those round trips overlap the bulk loads.
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

// x mod m for x >= 0, m > 0: a mask when m is a power of two (the usual window and slot
// counts), the 64-bit remainder otherwise.
__device__ inline int mod_index(int64_t x, int m) {
  return (m & (m - 1)) == 0 ? int(x & int64_t(m - 1)) : int(x % m);
}

// Registers a warp carries from load_scan to apply.
template <typename T, int ROWS, int NSC>
struct CommitRegs {
  uint4 raw[ROWS];                // this lane's 16-byte pieces of verify rows rg + j * rpi
  float g[Elem<T>::kVec];         // global sum (lanes of row group 0)
  float pr[NSC][Elem<T>::kVec];   // partial sums per scale (lanes of row group 0)
};

// Where the verify rows come from: the dense verify block [b][L][B+1][Hkv][D] ...
struct DenseVerify {
  const void* k;
  const void* v;
};
// ... or the target's paged KV cache, verify row i at the target's position len + i.
struct PagedVerify {
  ls_paged_kv kv;
};

// Loads a source needs before the scan (issued with the counters and token ids): the
// verify rows' slots when the caller passes an engine's slot mapping.
template <int ROWS>
__device__ inline void early_verify(const Dev&, const DenseVerify&, int, int, int, int64_t (&)[ROWS]) {}

template <int ROWS>
__device__ inline void early_verify(const Dev& p, const PagedVerify& s, int b, int rg, int rpi,
                                    int64_t (&slot)[ROWS]) {
  if (!s.kv.verify_slots) return;
  const int64_t* src = s.kv.verify_slots + int64_t(b) * (p.B + 1);
#pragma unroll
  for (int j = 0; j < ROWS; ++j) {
    const int i = rg + j * rpi;
    if (i <= p.B) slot[j] = __ldg(src + i);
  }
}

// This lane's 16-byte pieces of the retained verify rows 0..a (rows rg + j * rpi).
template <typename T, int ROWS>
__device__ inline void load_verify_rows(const Dev& p, const DenseVerify& s, int bl, int h, int t, int64_t, int a,
                                        int rg, int rpi, int cb, const int64_t (&)[ROWS], uint4 (&raw)[ROWS]) {
  const int64_t row_stride = int64_t(p.Hkv) * p.D;
  const T* src = static_cast<const T*>(t == 0 ? s.k : s.v) + int64_t(bl) * (p.B + 1) * row_stride +
                 int64_t(h) * p.D + cb;
#pragma unroll
  for (int j = 0; j < ROWS; ++j) {
    const int i = rg + j * rpi;
    if (i <= a) raw[j] = ld_nc_v4(src + int64_t(i) * row_stride);
  }
}

template <typename T, int ROWS>
__device__ inline void load_verify_rows(const Dev& p, const PagedVerify& s, int bl, int h, int t, int64_t len,
                                        int a, int rg, int rpi, int cb, const int64_t (&slot)[ROWS],
                                        uint4 (&raw)[ROWS]) {
  const int b = bl / p.L, l = bl - b * p.L;
  const char* base = static_cast<const char*>(t == 0 ? s.kv.k_layers[l] : s.kv.v_layers[l]);
  const int64_t col = (int64_t(h) * p.D + cb) * int64_t(sizeof(T));
  // the slots given, else every page lookup first, so the row loads leave in one round trip
  const char* rp[ROWS];
  const bool given = s.kv.verify_slots != nullptr;
#pragma unroll
  for (int j = 0; j < ROWS; ++j) {
    const int i = rg + j * rpi;
    rp[j] = i > a ? nullptr
                  : (given ? paged_slot(s.kv, base, slot[j], int(sizeof(T)), p.err)
                           : paged_row(s.kv, base, b, len + i, int(sizeof(T)), p.err));
  }
#pragma unroll
  for (int j = 0; j < ROWS; ++j)
    if (rg + j * rpi <= a) raw[j] = ld_nc_v4(rp[j] + col);
}

template <typename T, int ROWS, int NSC, typename Src>
__device__ inline void commit_load_scan(const Dev& p, int bl, int h, int t, int lane,
                                        const int32_t* __restrict__ draft, const int32_t* __restrict__ target,
                                        const Src& vsrc, CommitRegs<T, ROWS, NSC>& r,
                                        CommitScan& cs, const int32_t* __restrict__ given_a = nullptr) {
  constexpr int VEC = Elem<T>::kVec;
  const int b = bl / p.L;
  const int64_t* ctr = p.counters + int64_t(bl) * (1 + NSC);
  const int lpr = p.D / VEC;  // lanes per row: a power of two <= 32 (host-checked)
  const int rpi = 32 / lpr;   // rows per warp instruction
  const int c = lane & (lpr - 1), rg = lane / lpr;
  const int cb = c * VEC;
  const int64_t tile = int64_t(bl) * p.Hkv + h;

  int64_t early[ROWS];
  early_verify<ROWS>(p, vsrc, b, rg, rpi, early);
  const int64_t len = ctr[0];
  int64_t nseg[kMaxScales];
#pragma unroll
  for (int k = 0; k < kMaxScales; ++k) nseg[k] = k < NSC ? ctr[1 + k] : 0;
  bool mism[2] = {false, false};
  int a_given = 0;
  if (given_a) {  // the accepted count comes from the caller (stochastic acceptance)
    a_given = given_a[b];
    if (a_given < 0 || a_given > p.B) {
      if (lane == 0 && t == 0) set_err(p.err, LS_DEVERR_SAMPLE);
      a_given = a_given < 0 ? 0 : p.B;
    }
  } else {
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int i = 32 * w + lane;
      mism[w] = i < p.B && draft[int64_t(b) * p.B + i] != target[int64_t(b) * (p.B + 1) + i];
    }
  }
  // greedy acceptance: first i with draft[i] != target[i], else B
  const unsigned m0 = __ballot_sync(0xffffffffu, mism[0]);
  const unsigned m1 = __ballot_sync(0xffffffffu, mism[1]);
  const int a = given_a ? a_given : (m0 ? __ffs(m0) - 1 : (m1 ? 32 + __ffs(m1) - 1 : p.B));
  // scale k closes a segment this round exactly when its own distance to the next
  // boundary is <= Delta (then that distance equals the split row)
  unsigned closes = 0;
#pragma unroll
  for (int k = 0; k < NSC; ++k)
    if (p.scales[k] - (len - nseg[k] * p.scales[k]) <= a + 1) closes |= 1u << k;
  cs.a = a;
  cs.len = len;
  cs.newlen = len + a + 1;
#pragma unroll
  for (int k = 0; k < kMaxScales; ++k) cs.nseg[k] = nseg[k];
  cs.closes = closes;
  // the rest of the round's inputs: issued once a is known (only the retained rows are
  // read), so they share one round trip with the loads the caller issues next (the
  // boundary slice at verify row a)
  load_verify_rows<T, ROWS>(p, vsrc, bl, h, t, len, a, rg, rpi, cb, early, r.raw);
  if (rg == 0) {
    const float* gp = p.glob + (tile * 2 + t) * p.D + cb;
#pragma unroll
    for (int e = 0; e < VEC; e += 4) {
      const float4 v4 = *reinterpret_cast<const float4*>(gp + e);
      r.g[e] = v4.x; r.g[e + 1] = v4.y; r.g[e + 2] = v4.z; r.g[e + 3] = v4.w;
    }
#pragma unroll
    for (int k = 0; k < NSC; ++k) {
      const float* pp = p.part + ((tile * NSC + k) * 2 + t) * p.D + cb;
#pragma unroll
      for (int e = 0; e < VEC; e += 4) {
        const float4 v4 = *reinterpret_cast<const float4*>(pp + e);
        r.pr[k][e] = v4.x; r.pr[k][e + 1] = v4.y; r.pr[k][e + 2] = v4.z; r.pr[k][e + 3] = v4.w;
      }
    }
  }
}

template <typename T, int ROWS, int NSC>
__device__ inline void commit_apply(const Dev& p, int bl, int h, int t, int lane, CommitRegs<T, ROWS, NSC>& r,
                                    const CommitScan& cs) {
  using E = Elem<T>;
  constexpr int VEC = E::kVec;
  const int lpr = p.D / VEC;
  const int rpi = 32 / lpr;
  const int c = lane & (lpr - 1), rg = lane / lpr;
  const int cb = c * VEC;
  const int64_t tile = int64_t(bl) * p.Hkv + h;
  const int delta = cs.a + 1;
  const int c_split = int(p.scales[0] - (cs.len - cs.nseg[0] * p.scales[0]));

  T* kvt = reinterpret_cast<T*>(p.kv) + (tile * 2 + t) * int64_t(p.R) * p.D;
  float lo[VEC], hi[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) lo[e] = hi[e] = 0.f;
  const int ring0 = mod_index(cs.len, p.W);
#pragma unroll
  for (int j = 0; j < ROWS; ++j) {
    const int i = rg + j * rpi;
    if (i < delta) {
      int slot = ring0 + i;
      if (slot >= p.W) slot -= p.W;  // Delta <= W
      *reinterpret_cast<uint4*>(kvt + int64_t(slot) * p.D + cb) = r.raw[j];
      float f[VEC];
      E::to_f32(r.raw[j], f);
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
  if (rg != 0) return;
  float m[VEC];
  // global sum and its mean row
  float* gp = p.glob + (tile * 2 + t) * p.D + cb;
#pragma unroll
  for (int e = 0; e < VEC; ++e) r.g[e] += lo[e] + hi[e];
#pragma unroll
  for (int e = 0; e < VEC; e += 4)
    *reinterpret_cast<float4*>(gp + e) = make_float4(r.g[e], r.g[e + 1], r.g[e + 2], r.g[e + 3]);
  // mean rows are the attention's copy: one correctly rounded reciprocal per count
  const float inv_len = __frcp_rn(float(cs.newlen));
#pragma unroll
  for (int e = 0; e < VEC; ++e) m[e] = r.g[e] * inv_len;
  *reinterpret_cast<uint4*>(kvt + int64_t(p.R - 1) * p.D + cb) = E::from_f32(m);

#pragma unroll
  for (int k = 0; k < NSC; ++k) {
    const int sc = p.scales[k];
    float* pp = p.part + ((tile * NSC + k) * 2 + t) * p.D + cb;
    const bool completes = (cs.closes >> k) & 1u;
    const int64_t row0 = int64_t(p.W) + int64_t(k) * (p.slots + 1);
    if (completes) {
      const int slot = mod_index(cs.nseg[k], p.slots);
      const float inv_sc = __frcp_rn(float(sc));  // exact for power-of-two scales
#pragma unroll
      for (int e = 0; e < VEC; ++e) m[e] = (r.pr[k][e] + lo[e]) * inv_sc;
      float* sg = p.seg + (((tile * NSC + k) * p.slots + slot) * 2 + t) * p.D + cb;
#pragma unroll
      for (int e = 0; e < VEC; e += 4)
        *reinterpret_cast<float4*>(sg + e) = make_float4(m[e], m[e + 1], m[e + 2], m[e + 3]);
      *reinterpret_cast<uint4*>(kvt + (row0 + slot) * p.D + cb) = E::from_f32(m);
#pragma unroll
      for (int e = 0; e < VEC; ++e) r.pr[k][e] = hi[e];
    } else {  // no boundary crossed at this scale: every row extends the open segment
#pragma unroll
      for (int e = 0; e < VEC; ++e) r.pr[k][e] += lo[e] + hi[e];
    }
#pragma unroll
    for (int e = 0; e < VEC; e += 4)
      *reinterpret_cast<float4*>(pp + e) = make_float4(r.pr[k][e], r.pr[k][e + 1], r.pr[k][e + 2], r.pr[k][e + 3]);
    const int64_t cnt = cs.newlen - (cs.nseg[k] + (completes ? 1 : 0)) * int64_t(sc);
    const float inv_cnt = cnt > 0 ? __frcp_rn(float(cnt)) : 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) m[e] = r.pr[k][e] * inv_cnt;
    *reinterpret_cast<uint4*>(kvt + (row0 + p.slots) * p.D + cb) = E::from_f32(m);
  }
}

// The boundary view (Figure 2 caption (b)): the hidden vector at verify row a becomes the
// sequence-layer's boundary state. Each KV head's CTA copies its own 1/Hkv slice, so the
// copy is spread over the (sequence, layer)'s CTAs. Loads (after the scan) and stores
// (after the commit's own stores) are separate so the load round trip overlaps; a slice
// larger than kPieces pieces per thread is copied in a loop at the store instead.
// VEC-element pieces; hidden % VEC == 0.
template <typename T, int kPieces>
struct BoundarySlice {
  uint4 v[kPieces];
  int beg, end;
  bool staged;  // the slice fits in the registers
};

template <typename T, int kPieces>
__device__ inline void boundary_load(const Dev& p, int bl, int h, int a, int tid, int nthreads,
                                     const T* __restrict__ vh, BoundarySlice<T, kPieces>& s) {
  constexpr int VEC = Elem<T>::kVec;
  const int pieces = p.hidden / VEC;
  const int per = (pieces + p.Hkv - 1) / p.Hkv;
  s.beg = h * per;
  s.end = s.beg + per < pieces ? s.beg + per : pieces;
  s.staged = per <= kPieces * nthreads;
  if (!s.staged) return;
  const T* hrow = vh + (int64_t(bl) * (p.B + 1) + a) * p.hidden;
#pragma unroll
  for (int u = 0; u < kPieces; ++u) {
    const int x = s.beg + tid + u * nthreads;
    if (x < s.end) s.v[u] = ld_nc_v4(hrow + int64_t(x) * VEC);
  }
}

template <typename T, int kPieces>
__device__ inline void boundary_store(const Dev& p, int bl, int a, int tid, int nthreads,
                                      const T* __restrict__ vh, const BoundarySlice<T, kPieces>& s) {
  constexpr int VEC = Elem<T>::kVec;
  T* brow = reinterpret_cast<T*>(p.boundary) + int64_t(bl) * p.hidden;
  if (s.staged) {
#pragma unroll
    for (int u = 0; u < kPieces; ++u) {
      const int x = s.beg + tid + u * nthreads;
      if (x < s.end) *reinterpret_cast<uint4*>(brow + int64_t(x) * VEC) = s.v[u];
    }
    return;
  }
  const T* hrow = vh + (int64_t(bl) * (p.B + 1) + a) * p.hidden;
  for (int x0 = s.beg + tid; x0 < s.end; x0 += kPieces * nthreads) {
    uint4 v[kPieces];
#pragma unroll
    for (int u = 0; u < kPieces; ++u)
      if (x0 + u * nthreads < s.end) v[u] = ld_nc_v4(hrow + int64_t(x0 + u * nthreads) * VEC);
#pragma unroll
    for (int u = 0; u < kPieces; ++u)
      if (x0 + u * nthreads < s.end) *reinterpret_cast<uint4*>(brow + int64_t(x0 + u * nthreads) * VEC) = v[u];
  }
}

// rows of the verify block a lane may need: ceil((B + 1) / rows per warp instruction)
template <typename T>
__host__ __device__ inline int commit_rows_per_lane(int D, int B) {
  const int lpr = D / Elem<T>::kVec;
  return (B + 1 + (32 / lpr) - 1) / (32 / lpr);
}

}  // namespace ls
