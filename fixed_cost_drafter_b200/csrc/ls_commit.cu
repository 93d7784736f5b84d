// View extraction from the target's verification pass: LongSpark paper page,
// Figure 2 caption (a)-(b) and Figure 3 caption. One CTA of two warps per (sequence,
// layer, KV head); warp t runs the shared per-tensor body (ls_commit_body.cuh) for tensor t
// (0 = K, 1 = V). The head-0 CTA of a (sequence, layer) copies verify row a's hidden
// vectors into the boundary view, and the last of the (sequence, layer)'s CTAs to finish
// (an arrival counter) writes the new counters, after every CTA has read the old ones.
#include "ls_commit_body.cuh"

namespace ls {

template <typename T, int ROWS>
__global__ void __launch_bounds__(64)
commit_round_kernel(Dev p, const int32_t* __restrict__ draft, const int32_t* __restrict__ target,
                    const T* __restrict__ vk, const T* __restrict__ vv,
                    const T* __restrict__ vh, int32_t* __restrict__ accept_len,
                    int32_t* __restrict__ next_token) {
  // the attention kernel of ls_round may be scheduled now: it waits on the device for
  // this grid's writes before it reads any state
  allow_dependent_launch();
  const int bl = blockIdx.x / p.Hkv, h = blockIdx.x - bl * p.Hkv;
  const int b = bl / p.L, l = bl - b * p.L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  CommitScan cs;
  commit_tensor<T, ROWS>(p, bl, h, warp, lane, draft, target, warp == 0 ? vk : vv, cs);

  // boundary state: this KV head's slice of the hidden vector at verify row a
  copy_boundary_slice<T, 4>(p, bl, h, cs.a, threadIdx.x, blockDim.x, vh);

  __syncthreads();  // both warps have read the counters
  if (threadIdx.x == 0) {
    // the last KV-head CTA of this (sequence, layer) to arrive writes the new counters:
    // every other one has read the old counters before its own arrival
    const int before = atomicAdd(p.arrive + bl, 1);
    if (before == p.Hkv - 1) {
      int64_t* ctr = p.counters + int64_t(bl) * (1 + p.nsc);
      p.arrive[bl] = 0;
      ctr[0] = cs.newlen;
#pragma unroll
      for (int k = 0; k < kMaxScales; ++k)
        if (k < p.nsc) ctr[1 + k] = cs.nseg[k] + ((cs.closes >> k) & 1u);
      if (l == 0) {
        accept_len[b] = cs.a;
        next_token[b] = target[int64_t(b) * (p.B + 1) + cs.a];
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
  const int rows = commit_rows_per_lane<T>(p.D, p.B);
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
