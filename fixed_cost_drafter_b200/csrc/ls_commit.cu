// View extraction from the target's verification pass: LongSpark paper page,
// Figure 2 caption (a)-(b) and Figure 3 caption. One CTA of two warps per (sequence,
// layer, KV head); warp t runs the per-tensor body (ls_commit_body.cuh) for tensor t
// (0 = K, 1 = V). Every KV head's CTA copies its slice of verify row a's hidden vector into
// the boundary view, and the last of the (sequence, layer)'s CTAs to arrive (an arrival
// counter) writes the new counters, after every CTA has read the old ones. The scan needs
// only the counters and token ids; the bulk inputs, the slice's loads and the arrival are
// all issued right after it, in one round trip. The verify rows come from the dense verify
// block or, read in place, from the target's paged KV cache (one more dependent lookup:
// the block table entry of each retained position).
#include "ls_commit_body.cuh"

namespace ls {

template <typename T, int ROWS, int NSC, typename Src>
__global__ void __launch_bounds__(64)
commit_round_kernel(Dev p, const int32_t* __restrict__ draft, const int32_t* __restrict__ target,
                    const Src src, const T* __restrict__ vh, int32_t* __restrict__ accept_len,
                    int32_t* __restrict__ next_token, const int32_t* __restrict__ given_a) {
  const int bl = blockIdx.x / p.Hkv, h = blockIdx.x - bl * p.Hkv;
  const int b = bl / p.L, l = bl - b * p.L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  CommitRegs<T, ROWS, NSC> r;
  CommitScan cs;
  commit_load_scan<T, ROWS, NSC>(p, bl, h, warp, lane, draft, target, src, r, cs, given_a);
  // boundary state: this KV head's slice of the hidden vector at verify row a (loads now,
  // stores after the commit's own)
  BoundarySlice<T, 2> bs;
  boundary_load<T, 2>(p, bl, h, cs.a, threadIdx.x, 64, vh, bs);
  // the attention kernel of ls_round may be scheduled now: it waits on the device for
  // this grid's writes before it reads any state. Triggered once this CTA's loads are in
  // flight, not at entry: attention CTAs made resident earlier slowed the commit's
  // dependent loads (counters, then the rows) after a cold L2 by 2 to 10 us per round.
  allow_dependent_launch();
  __syncthreads();  // both warps have read the old counters
  // the last of the (sequence, layer)'s CTAs to arrive writes the new counters: every
  // other one has read the old counters before its own arrival
  int before = 0;
  if (threadIdx.x == 0) before = atomicAdd(p.arrive + bl, 1);
  commit_apply<T, ROWS, NSC>(p, bl, h, warp, lane, r, cs);
  boundary_store<T, 2>(p, bl, cs.a, threadIdx.x, 64, vh, bs);
  if (threadIdx.x == 0 && before == p.Hkv - 1) {
    int64_t* ctr = p.counters + int64_t(bl) * (1 + NSC);
    p.arrive[bl] = 0;
    ctr[0] = cs.newlen;
#pragma unroll
    for (int k = 0; k < NSC; ++k) ctr[1 + k] = cs.nseg[k] + ((cs.closes >> k) & 1u);
    if (l == 0 && !given_a) {  // with given counts the caller has the tokens
      accept_len[b] = cs.a;
      next_token[b] = target[int64_t(b) * (p.B + 1) + cs.a];
    }
  }
}

template <typename T, int ROWS, int NSC, typename Src>
static void launch_commit_t(const Dev& p, const int32_t* draft, const int32_t* target, const Src& src,
                            const void* vh, int32_t* accept_len, int32_t* next_token, const int32_t* given_a,
                            cudaStream_t stream) {
  commit_round_kernel<T, ROWS, NSC, Src><<<p.b * p.L * p.Hkv, 64, 0, stream>>>(
      p, draft, target, src, static_cast<const T*>(vh), accept_len, next_token, given_a);
}

template <typename T, int ROWS, typename Src>
static void launch_commit_rows(const Dev& p, const int32_t* draft, const int32_t* target, const Src& src,
                               const void* vh, int32_t* accept_len, int32_t* next_token, const int32_t* given_a,
                               cudaStream_t stream) {
  switch (p.nsc) {  // the scale count is a template argument: only live scale code is compiled
    case 1: launch_commit_t<T, ROWS, 1>(p, draft, target, src, vh, accept_len, next_token, given_a, stream); break;
    case 2: launch_commit_t<T, ROWS, 2>(p, draft, target, src, vh, accept_len, next_token, given_a, stream); break;
    case 3: launch_commit_t<T, ROWS, 3>(p, draft, target, src, vh, accept_len, next_token, given_a, stream); break;
    default: launch_commit_t<T, ROWS, 4>(p, draft, target, src, vh, accept_len, next_token, given_a, stream); break;
  }
}

// rows per lane: bf16 rows are 16 lanes wide (2 rows per warp instruction), fp32 rows 32
// lanes; B <= 32 (host-checked)
template <typename T, typename Src>
static void launch_commit_dt(const Dev& p, const int32_t* draft, const int32_t* target, const Src& src,
                             const void* vh, int32_t* accept_len, int32_t* next_token, const int32_t* given_a,
                             cudaStream_t stream) {
  const int rows = commit_rows_per_lane<T>(p.D, p.B);
  if (rows <= 9) launch_commit_rows<T, 9>(p, draft, target, src, vh, accept_len, next_token, given_a, stream);
  else if (rows <= 17) launch_commit_rows<T, 17>(p, draft, target, src, vh, accept_len, next_token, given_a, stream);
  else launch_commit_rows<T, 33>(p, draft, target, src, vh, accept_len, next_token, given_a, stream);
}

template <typename Src>
static cudaError_t launch_commit_src(const Dev& p, const int32_t* draft, const int32_t* target, const Src& src,
                                     const void* vh, int32_t* accept_len, int32_t* next_token,
                                     const int32_t* given_a, cudaStream_t stream) {
  if (p.dtype == LS_BF16)
    launch_commit_dt<__nv_bfloat16>(p, draft, target, src, vh, accept_len, next_token, given_a, stream);
  else
    launch_commit_dt<float>(p, draft, target, src, vh, accept_len, next_token, given_a, stream);
  return cudaGetLastError();
}

cudaError_t launch_commit(const Dev& p, const int32_t* draft, const int32_t* target, const void* vk,
                          const void* vv, const void* vh, int32_t* accept_len, int32_t* next_token,
                          const int32_t* given_a, cudaStream_t stream) {
  return launch_commit_src(p, draft, target, DenseVerify{vk, vv}, vh, accept_len, next_token, given_a, stream);
}

cudaError_t launch_commit_paged(const Dev& p, const int32_t* draft, const int32_t* target, const ls_paged_kv& kv,
                                const void* vh, int32_t* accept_len, int32_t* next_token, const int32_t* given_a,
                                cudaStream_t stream) {
  return launch_commit_src(p, draft, target, PagedVerify{kv}, vh, accept_len, next_token, given_a, stream);
}

}  // namespace ls
