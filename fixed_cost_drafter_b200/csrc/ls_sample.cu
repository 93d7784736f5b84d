// Stochastic acceptance for sampled decoding (T > 0): the pages compare greedy decoding
// (Table 3, T = 0) with sampled decoding (Table 1) but print no acceptance rule, so this
// is standard speculative sampling (Leviathan, Kalman and Matias 2023; Chen et al. 2023):
// draft i of a block is kept while u_i * q_i(d_i) < p_i(d_i) (fp32 product and compare),
// and the next token is drawn from max(0, p_a - q_a) after a rejection at position a (from
// p_a itself when that residual has no mass: speculative sampling emits samples of the
// target's distribution), or from p_B after B acceptances, by inverse CDF in vocabulary
// order with the draw u_B. A row drawn from that has no mass sets LS_DEVERR_SAMPLE.
//
// Grid (vocabulary chunks of 8192, sequences), 256 threads. Every CTA of a sequence makes
// the B acceptance tests itself (2 B gathers) and sums the draw's weights over its chunk:
// per segment of 128 entries (64 segments: sub-block m of 1024 entries, one float4 per
// thread, warp w's 128 of them) a fixed tree, and the chunk's total a fixed tree over its
// segments; it leaves both in the arena. The last CTA of the sequence to arrive (a counter
// in the arena, reset by that CTA; nobody waits) scans the chunk totals in order for the
// chunk holding u_B times the total, then that chunk's segment sums for the segment, and
// one warp re-reads the segment's 128 entries from L2 for the entry. HBM traffic: the rows
// of the draw (one, or two after a rejection) once.
#include "ls_common.cuh"

namespace ls {

namespace {

constexpr int kSampleThreads = 256;
constexpr int kSub = kSampleThreads * 4;    // entries per sub-block (one float4 per thread)
constexpr int kSubs = kSampleChunk / kSub;  // sub-blocks per chunk

struct SampleArgs {
  const int32_t* draft;   // [b][B]
  const float* q;         // [b][B][V]
  const float* p;         // [b][B+1][V]
  const float* u;         // [b][B+1]
  int32_t* accept_len;    // [b]
  int32_t* next_token;    // [b]
  int32_t V, nchunks;
};

// Weights of entries j..j+3 (j a multiple of 4, V a multiple of 4): max(0, p - q) after a
// rejection (qrow set), else p; entries past the vocabulary weigh 0.
__device__ inline float4 weights4(const float* prow, const float* qrow, int j, int V) {
  if (j >= V) return make_float4(0.f, 0.f, 0.f, 0.f);
  // (plain loads: the drawn chunk is read again from L2 by the sequence's last CTA)
  float4 w = *reinterpret_cast<const float4*>(prow + j);
  if (qrow) {
    const float4 q = *reinterpret_cast<const float4*>(qrow + j);
    w.x = fmaxf(0.f, w.x - q.x);
    w.y = fmaxf(0.f, w.y - q.y);
    w.z = fmaxf(0.f, w.z - q.z);
    w.w = fmaxf(0.f, w.w - q.w);
  }
  return w;
}
__device__ inline float sum4(const float4& w) { return (w.x + w.y) + (w.z + w.w); }

// Segment j = 8 m + w of a chunk: the 128 entries [1024 m + 128 w, +128) that warp w's
// float4 loads of sub-block m cover. A chunk's 64 segment sums, in entry order, and its
// total (a fixed tree over them) are what the chunk's CTA leaves for the sequence's last CTA.
constexpr int kSegs = kSubs * (kSampleThreads / 32);  // 64
static_assert(kSegs == 64, "the segment scan covers 64 entries with two warps");

// The segment sums of chunk c into seg[64] (every thread calls it; ends with a barrier).
__device__ inline void chunk_segments(const float* prow, const float* qrow, int c, int V, float* seg) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int base = c * kSampleChunk + 4 * threadIdx.x;
  float r[kSubs];
#pragma unroll
  for (int m = 0; m < kSubs; ++m) r[m] = sum4(weights4(prow, qrow, base + m * kSub, V));
#pragma unroll
  for (int m = 0; m < kSubs; ++m)
#pragma unroll
    for (int o = 16; o; o >>= 1) r[m] += __shfl_xor_sync(0xffffffffu, r[m], o);
  if (lane == 0)
#pragma unroll
    for (int m = 0; m < kSubs; ++m) seg[m * (kSampleThreads / 32) + warp] = r[m];
  __syncthreads();
}

// The total of 64 segment sums: a fixed tree (pairs j, j + 32, then across the warp). Called
// by one whole warp; every lane gets it.
__device__ inline float segments_total(const float* seg) {
  const int lane = threadIdx.x & 31;
  float v = seg[lane] + seg[lane + 32];
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The first of n <= 64 sums (in order) whose running sum passes t: t = x * (their total)
// when `fraction`, else t = x. When rounding leaves none (or t is infinite), the last with
// mass, and *rem_out infinite; *idx_out -1 when none has mass. *rem_out otherwise gets t
// minus the sums before the one found. The first two warps scan; every thread calls it
// (ends with a barrier).
__device__ inline void find_first(const float* vals, int n, float x, bool fraction, float* sh, float* scratch,
                                  int* idx_out, float* rem_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < 2) {
    const int k = threadIdx.x;
    const float v = k < n ? vals[k] : 0.f;
    float inc = v;  // inclusive prefix within the warp, in order
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) sh[warp] = inc;
    asm volatile("bar.sync 1, 64;" ::: "memory");  // the two warps' totals
    if (warp == 1) inc += sh[0];
    const float z = sh[0] + sh[1];
    const float t = fraction ? x * z : x;
    const unsigned hit = __ballot_sync(0xffffffffu, z > 0.f && k < n && inc > t);
    const unsigned mass = __ballot_sync(0xffffffffu, k < n && v > 0.f);
    if (lane == 0) {
      scratch[warp] = __int_as_float(int(hit));
      scratch[2 + warp] = __int_as_float(int(mass));
    }
    asm volatile("bar.sync 1, 64;" ::: "memory");
    const unsigned h0 = __float_as_int(scratch[0]), h1 = __float_as_int(scratch[1]);
    const unsigned m0 = __float_as_int(scratch[2]), m1 = __float_as_int(scratch[3]);
    int idx = h0 ? __ffs(int(h0)) - 1 : (h1 ? 32 + __ffs(int(h1)) - 1 : -1);
    bool force_last = false;
    if (idx < 0 && (m0 | m1)) {
      idx = m1 ? 63 - __clz(int(m1)) : 31 - __clz(int(m0));
      force_last = true;
    }
    if (k == idx) {
      *idx_out = idx;
      *rem_out = force_last ? INFINITY : t - (inc - v);
    }
    if (threadIdx.x == 0 && idx < 0) *idx_out = -1;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSampleThreads) sample_kernel(const Dev p, const SampleArgs s) {
  const int c = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float sh[kSampleThreads / 32];
  __shared__ float scratch[4];
  __shared__ float csum_s[kSampleMaxChunks];
  __shared__ float seg_s[kSegs];
  __shared__ int a_s, last_s, cstar_s, sstar_s;
  __shared__ float rem_s, rem2_s;

  // the accepted count: first position whose test fails (B <= 32: one warp)
  if (warp == 0) {
    bool rej = false;
    if (lane < p.B) {
      const int d = s.draft[b * p.B + lane];
      if (d < 0 || d >= s.V) {
        rej = true;
        if (c == 0) set_err(p.err, LS_DEVERR_SAMPLE);
      } else {
        const float qd = s.q[(int64_t(b) * p.B + lane) * s.V + d];
        const float pd = s.p[(int64_t(b) * (p.B + 1) + lane) * s.V + d];
        rej = !(__fmul_rn(s.u[b * (p.B + 1) + lane], qd) < pd);
      }
    }
    const unsigned m = __ballot_sync(0xffffffffu, rej);
    if (lane == 0) a_s = m ? __ffs(int(m)) - 1 : p.B;
  }
  __syncthreads();
  const int a = a_s;
  const float* prow = s.p + (int64_t(b) * (p.B + 1) + a) * s.V;
  const float* qrow = a < p.B ? s.q + (int64_t(b) * p.B + a) * s.V : nullptr;  // null: draw from p

  // this chunk's share of the draw's mass: its 64 segment sums and their total
  float* seg_g = p.samp_seg + (int64_t(b) * kSampleMaxChunks + c) * kSegs;
  chunk_segments(prow, qrow, c, s.V, seg_s);
  if (threadIdx.x < kSegs) seg_g[threadIdx.x] = seg_s[threadIdx.x];
  if (warp == 0) {
    const float tot = segments_total(seg_s);
    if (lane == 0) p.samp_part[b * kSampleMaxChunks + c] = tot;
  }
  __threadfence();  // (the segment sums and the total are visible before the arrival)
  __syncthreads();
  if (threadIdx.x == 0) last_s = atomicAdd(p.samp_count + b, 1) == s.nchunks - 1;
  __syncthreads();
  if (!last_s) return;

  // The sequence's last CTA: the chunk holding u_B times the total, then its segment, then
  // the entry (one warp re-reads the segment's 128 entries from L2).
  __threadfence();
  if (threadIdx.x < kSampleMaxChunks)
    csum_s[threadIdx.x] =
        int(threadIdx.x) < s.nchunks ? __ldcg(p.samp_part + b * kSampleMaxChunks + threadIdx.x) : 0.f;
  if (threadIdx.x == 0) p.samp_count[b] = 0;  // zero again for the next call
  __syncthreads();
  const float ub = s.u[b * (p.B + 1) + p.B];
  find_first(csum_s, s.nchunks, ub, true, sh, scratch, &cstar_s, &rem_s);
  bool local = false;  // the chosen chunk's segment sums are computed here, not loaded
  if (cstar_s < 0 && qrow != nullptr) {
    // The residual has no mass (p_a <= q_a everywhere: equal rows up to rounding, or a
    // draft neither row gives mass): the token is drawn from the target's row p_a itself,
    // whose chunk sums this CTA makes in the order the chunk CTAs use.
    qrow = nullptr;
    local = true;
    for (int c2 = 0; c2 < s.nchunks; ++c2) {
      chunk_segments(prow, nullptr, c2, s.V, seg_s);
      if (warp == 0) {
        const float tot = segments_total(seg_s);
        if (lane == 0) csum_s[c2] = tot;
      }
      __syncthreads();
    }
    find_first(csum_s, s.nchunks, ub, true, sh, scratch, &cstar_s, &rem_s);
  }
  if (cstar_s < 0) {  // the row drawn from has no mass: not a distribution
    if (threadIdx.x == 0) {
      s.accept_len[b] = a;
      s.next_token[b] = 0;
      set_err(p.err, LS_DEVERR_SAMPLE);
    }
    return;
  }
  const int cs = cstar_s;
  if (local) {
    chunk_segments(prow, nullptr, cs, s.V, seg_s);
  } else {
    if (threadIdx.x < kSegs)
      seg_s[threadIdx.x] = __ldcg(p.samp_seg + (int64_t(b) * kSampleMaxChunks + cs) * kSegs + threadIdx.x);
    __syncthreads();
  }
  find_first(seg_s, kSegs, rem_s, false, sh, scratch, &sstar_s, &rem2_s);
  if (warp == 0) {
    // (the chunk has mass, so some segment has: sstar_s >= 0)
    const int sg = sstar_s < 0 ? 0 : sstar_s;
    const int j0 = cs * kSampleChunk + (sg / (kSampleThreads / 32)) * kSub + (sg % (kSampleThreads / 32)) * 128;
    const int pos = j0 + 4 * lane;
    const float4 w = weights4(prow, qrow, pos, s.V);
    const float ls = sum4(w);
    float inc = ls;  // running sum over the lanes, in order
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    float excl = __shfl_up_sync(0xffffffffu, inc, 1);
    if (lane == 0) excl = 0.f;
    float rem = rem2_s;
    const unsigned hit = __ballot_sync(0xffffffffu, inc > rem);
    const unsigned mass = __ballot_sync(0xffffffffu, ls > 0.f);
    int ln = hit ? __ffs(int(hit)) - 1 : -1;
    if (ln < 0) {  // rounding: the last lane with mass
      ln = mass ? 31 - __clz(int(mass)) : 0;
      rem = INFINITY;
    }
    if (lane == ln) {
      const float e4[4] = {w.x, w.y, w.z, w.w};
      float run = excl;
      int pick = -1;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        run += e4[e];
        if (pick < 0 && run > rem && e4[e] > 0.f) pick = e;
      }
      if (pick < 0)  // rounding inside the four: their last entry with mass
        for (int e = 3; e >= 0 && pick < 0; --e)
          if (e4[e] > 0.f) pick = e;
      s.accept_len[b] = a;
      s.next_token[b] = pos + (pick < 0 ? 0 : pick);
    }
  }
}

}  // namespace

cudaError_t launch_sample(const Dev& p, const int32_t* draft, const float* q, const float* pr, int vocab,
                          const float* u, int32_t* accept_len, int32_t* next_token, cudaStream_t stream) {
  SampleArgs s{draft, q, pr, u, accept_len, next_token, vocab, (vocab + kSampleChunk - 1) / kSampleChunk};
  sample_kernel<<<dim3(s.nchunks, p.b), kSampleThreads, 0, stream>>>(p, s);
  return cudaGetLastError();
}

}  // namespace ls
