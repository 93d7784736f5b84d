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
// the B acceptance tests itself (2 B gathers) and sums the draw's weights over its chunk
// in a fixed order: sub-block m of 1024 entries, one float4 per thread, sub-blocks in
// order, then a tree over the threads. The last CTA of the sequence to arrive (a counter
// in the arena, reset by that CTA; nobody waits) adds the chunk sums in order, finds the
// chunk, then the sub-block, thread and entry holding the draw. HBM traffic: the rows of
// the draw (one, or two after a rejection) once, plus the drawn chunk again.
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

// Sum over the CTA (warp trees, then the 8 warp sums in order); every thread gets it.
__device__ inline float block_sum(float x, float* sh) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = x;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kSampleThreads / 32; ++w) t += sh[w];
  return t;
}

// Exclusive prefix of x over the threads in order; *total gets the sum of all.
__device__ inline float block_exclusive(float x, float* sh, float* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  __syncthreads();
  if (lane == 31) sh[warp] = inc;
  __syncthreads();
  float before = 0.f, all = 0.f;
#pragma unroll
  for (int w = 0; w < kSampleThreads / 32; ++w) {
    if (w < warp) before += sh[w];
    all += sh[w];
  }
  *total = all;
  return before + inc - x;
}

// The chunk holding the draw: the first chunk whose running sum (chunks in order) passes
// t = u * total, or the last chunk with mass when rounding leaves none. The first two warps
// scan the nchunks <= 64 sums in csum; *cstar gets the chunk (-1: no mass at all) and *rem
// the part of t left inside it (infinity in the rounding case). Every thread calls it.
__device__ inline void find_chunk(const float* csum, int nchunks, float u, float* sh, float* scratch, int* cstar_out,
                                  float* rem_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < 2) {
    const int k = threadIdx.x;
    const float v = k < nchunks ? csum[k] : 0.f;
    float inc = v;  // inclusive prefix within the warp, in chunk order
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) sh[warp] = inc;
    asm volatile("bar.sync 1, 64;" ::: "memory");  // the two warps' totals
    if (warp == 1) inc += sh[0];
    const float z = sh[0] + sh[1];
    const float t = u * z;
    const unsigned hit = __ballot_sync(0xffffffffu, z > 0.f && k < nchunks && inc > t);
    const unsigned mass = __ballot_sync(0xffffffffu, k < nchunks && v > 0.f);
    if (lane == 0) {
      scratch[warp] = __int_as_float(int(hit));
      scratch[2 + warp] = __int_as_float(int(mass));
    }
    asm volatile("bar.sync 1, 64;" ::: "memory");
    const unsigned h0 = __float_as_int(scratch[0]), h1 = __float_as_int(scratch[1]);
    const unsigned m0 = __float_as_int(scratch[2]), m1 = __float_as_int(scratch[3]);
    int cstar = h0 ? __ffs(int(h0)) - 1 : (h1 ? 32 + __ffs(int(h1)) - 1 : -1);
    bool force_last = false;
    if (cstar < 0 && z > 0.f) {
      cstar = m1 ? 63 - __clz(int(m1)) : 31 - __clz(int(m0));
      force_last = true;
    }
    if (k == cstar) {
      *cstar_out = cstar;
      *rem_out = force_last ? INFINITY : t - (inc - v);
    }
    if (threadIdx.x == 0 && cstar < 0) *cstar_out = -1;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSampleThreads) sample_kernel(const Dev p, const SampleArgs s) {
  const int c = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float sh[kSampleThreads / 32];
  __shared__ float sub_tot[kSubs];
  __shared__ float sub_part[kSampleThreads / 32][kSubs];
  __shared__ float csum_s[kSampleMaxChunks];
  __shared__ int a_s, last_s, cstar_s, found_s, lastpos_s;
  __shared__ float rem_s;

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

  // this chunk's share of the draw's mass
  {
    const int base = c * kSampleChunk + 4 * threadIdx.x;
    float acc = 0.f;
#pragma unroll
    for (int m = 0; m < kSubs; ++m) acc += sum4(weights4(prow, qrow, base + m * kSub, s.V));
    const float tot = block_sum(acc, sh);
    if (threadIdx.x == 0) {
      p.samp_part[b * kSampleMaxChunks + c] = tot;
      __threadfence();
      last_s = atomicAdd(p.samp_count + b, 1) == s.nchunks - 1;
    }
    __syncthreads();
    if (!last_s) return;
  }

  // the sequence's last CTA: the chunk sums (loaded at once, chunk k by thread k), then
  // the chunk holding u_B * total
  __threadfence();
  if (threadIdx.x < kSampleMaxChunks)
    csum_s[threadIdx.x] =
        int(threadIdx.x) < s.nchunks ? __ldcg(p.samp_part + b * kSampleMaxChunks + threadIdx.x) : 0.f;
  if (threadIdx.x == 0) p.samp_count[b] = 0;  // zero again for the next call
  __syncthreads();
  const float ub = s.u[b * (p.B + 1) + p.B];
  find_chunk(csum_s, s.nchunks, ub, sh, sub_tot, &cstar_s, &rem_s);
  if (cstar_s < 0 && qrow != nullptr) {
    // The residual has no mass (p_a <= q_a everywhere: equal rows up to rounding, or a
    // draft neither row gives mass): the token is drawn from the target's row p_a itself,
    // whose chunk sums this CTA makes in the order the chunk CTAs use.
    qrow = nullptr;
    for (int c2 = 0; c2 < s.nchunks; ++c2) {
      const int base = c2 * kSampleChunk + 4 * threadIdx.x;
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < kSubs; ++m) acc += sum4(weights4(prow, nullptr, base + m * kSub, s.V));
      const float tot = block_sum(acc, sh);
      if (threadIdx.x == 0) csum_s[c2] = tot;
    }
    __syncthreads();
    find_chunk(csum_s, s.nchunks, ub, sh, sub_tot, &cstar_s, &rem_s);
  }
  if (cstar_s < 0) {  // the row drawn from has no mass: not a distribution
    if (threadIdx.x == 0) {
      s.accept_len[b] = a;
      s.next_token[b] = 0;
      set_err(p.err, LS_DEVERR_SAMPLE);
    }
    return;
  }

  // sub-block and entry: the first entry whose running sum in the chunk passes rem
  const int cbase = cstar_s * kSampleChunk;
  float4 w[kSubs];
  float ws[kSubs];
#pragma unroll
  for (int m = 0; m < kSubs; ++m) {
    w[m] = weights4(prow, qrow, cbase + m * kSub + 4 * threadIdx.x, s.V);
    ws[m] = sum4(w[m]);
  }
  {
    // the 8 sub-block sums in one round: warp trees, then the warps' partials in order
    float r[kSubs];
#pragma unroll
    for (int m = 0; m < kSubs; ++m) {
      r[m] = ws[m];
#pragma unroll
      for (int o = 16; o; o >>= 1) r[m] += __shfl_xor_sync(0xffffffffu, r[m], o);
    }
    if (lane == 0)
#pragma unroll
      for (int m = 0; m < kSubs; ++m) sub_part[warp][m] = r[m];
    if (threadIdx.x == 0) {
      found_s = 0x7fffffff;
      lastpos_s = -1;
    }
    __syncthreads();
    if (threadIdx.x < kSubs) {
      float t = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < kSampleThreads / 32; ++w2) t += sub_part[w2][threadIdx.x];
      sub_tot[threadIdx.x] = t;
    }
    __syncthreads();
  }
  float rem = rem_s;
  int mstar = -1;
  for (int m = 0; m < kSubs && mstar < 0; ++m) {
    if (sub_tot[m] > rem) mstar = m;
    else rem -= sub_tot[m];
  }
  if (mstar < 0) {  // rounding: the last sub-block with mass, its last entry with mass
    for (int m = kSubs - 1; m >= 0 && mstar < 0; --m)
      if (sub_tot[m] > 0.f) mstar = m;
    if (mstar < 0) mstar = 0;  // (the chunk had mass in the first pass: not reached)
    rem = INFINITY;
  }
  float4 wm = w[0];
  float wsm = ws[0];
#pragma unroll
  for (int m = 1; m < kSubs; ++m)
    if (m == mstar) { wm = w[m]; wsm = ws[m]; }
  float total;
  const float excl = block_exclusive(wsm, sh, &total);
  const int pos0 = cbase + mstar * kSub + 4 * threadIdx.x;
  const float e4[4] = {wm.x, wm.y, wm.z, wm.w};
  if (excl <= rem && rem < excl + wsm) {  // this thread's four entries hold the draw
    float run = excl;
    int pick = -1;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      run += e4[e];
      if (pick < 0 && run > rem && e4[e] > 0.f) pick = e;
    }
    if (pick < 0)  // rounding inside the four: their last entry with mass (wsm > 0 here)
      for (int e = 3; e >= 0 && pick < 0; --e)
        if (e4[e] > 0.f) pick = e;
    atomicMin(&found_s, pos0 + pick);
  }
  // fallback for rounding at the end of the sub-block: its last entry with mass
#pragma unroll
  for (int e = 3; e >= 0; --e)
    if (e4[e] > 0.f) { atomicMax(&lastpos_s, pos0 + e); break; }
  __syncthreads();
  if (threadIdx.x == 0) {
    s.accept_len[b] = a;
    const int tok = found_s != 0x7fffffff ? found_s : lastpos_s;
    s.next_token[b] = tok >= 0 ? tok : 0;
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
