// The drafter's projections ahead of its attention: boundary keys/values from the boundary
// hidden vectors, block queries from the drafter's block inputs (LongSpark paper page,
// Figure 2 caption (c): the drafter uses the views; its projections are not described,
// the reading is a plain linear map per tapped layer). Both are dense contractions over
// the hidden size, so they run on the 5th-generation tensor cores:
//   Y[rows][n] = sum_k W[l][n][k] X[rows][l][k]   (bf16 in, fp32 accumulate, bf16 out)
// with the weights as the MMA's A operand (M = 128 weight rows per unit, K-major) and the
// activations as its B operand (N = up to 256 activation rows, K-major): the weights
// stream through once, the few activation rows come from L2.
//
// Persistent kernel, 6 warps: warp 0 TMA producer (a ring of 4 stages, each 64 hidden
// entries of the unit's 128 weight rows and of its activation rows, 128-byte swizzle),
// warp 1 TMEM allocator and MMA issuer (double-buffered accumulator, 2 x 256 columns),
// warps 2-5 epilogue (one TMEM subpartition each: a thread owns one weight row n and
// writes its column of outputs). Units: (problem, layer, 128-row weight tile, activation
// tile), queries first; CTA c takes units c, c + grid, ... Every wait is bounded.
#include "ls_tc.cuh"

namespace ls {

namespace {

constexpr int kPThreads = 192;
constexpr int kPStages = 4;
constexpr int kPKStep = 64;                          // hidden entries per stage
constexpr int kPTileN = 128;                         // weight rows per unit (MMA M)
constexpr int kPMaxAct = 256;                        // activation rows per unit (MMA N)
constexpr int kPABytes = kPTileN * kPKStep * 2;      // 16 KB
constexpr int kPBBytes = kPMaxAct * kPKStep * 2;     // 32 KB
constexpr int kPStageBytes = kPABytes + kPBBytes;
constexpr int kPSmemBytes = kPStages * kPStageBytes + 1024;
constexpr uint32_t kPTmemCols = 512;

struct PProblem {
  int32_t n_out;         // weight rows (output columns) per layer, a multiple of 128
  int32_t rows_per_seq;  // activation rows per sequence and layer: 1 (boundary) or B (block)
  int32_t seq_per_unit;  // sequences per activation tile
  int32_t load_rows;     // activation rows of a tile's box: seq_per_unit * rows_per_seq
  int32_t act_rows;      // the MMA's N: load_rows rounded up to 16 (the rows past load_rows
                         // are stale shared memory feeding accumulator columns never stored)
  int32_t m_tiles;       // activation tiles: ceil(b / seq_per_unit)
  int32_t n_units;       // L * (n_out / 128) * m_tiles
  int32_t is_4d;         // X tensor map is 4-D (block rows) or 3-D (boundary)
  __nv_bfloat16* y;      // [b][L][rows_per_seq][n_out]
};

struct PArgs {
  PProblem pr[2];
  int32_t b, L, k_steps;
  int32_t n_units;
  int32_t* err;
};

struct PBars {
  uint64_t full[kPStages], empty[kPStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;  // after an abort: the MMAs issued so far have completed
  uint32_t tmem_base;
  uint32_t abort;
};

struct PUnit {
  int p, l, nt, mt;
};

__device__ inline PUnit unit_of(const PArgs& a, int u) {
  PUnit r;
  r.p = u < a.pr[0].n_units ? 0 : 1;
  if (r.p) u -= a.pr[0].n_units;
  const int nts = a.pr[r.p].n_out / kPTileN;
  r.nt = u % nts;
  u /= nts;
  r.l = u % a.L;
  r.mt = u / a.L;
  return r;
}

__device__ inline bool pwait(PBars& s, uint64_t* bar, uint32_t parity, int32_t* err) {
#pragma unroll 1
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023) == 1023 && *reinterpret_cast<volatile uint32_t*>(&s.abort)) return false;
  }
  set_err(err, LS_DEVERR_WAIT_TIMEOUT);
  *reinterpret_cast<volatile uint32_t*>(&s.abort) = 1;
  return false;
}

__global__ void __launch_bounds__(kPThreads, 1)
prologue_kernel(const PArgs a, const __grid_constant__ CUtensorMap w0, const __grid_constant__ CUtensorMap x0,
                const __grid_constant__ CUtensorMap w1, const __grid_constant__ CUtensorMap x1) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ PBars s;
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_mine = int(blockIdx.x) < a.n_units ? (a.n_units - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPStages; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&s.acc_full[i], 1); mbar_init(&s.acc_empty[i], 128); }
    mbar_init(&s.drain, 1);
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s.tmem_base)),
                 "r"(kPTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  int issued = 0;  // producer: copies issued (for the drain after an abort)

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_map(&w0);
      prefetch_map(&x0);
      prefetch_map(&w1);
      prefetch_map(&x1);
      bool ok = true;
      int k = 0;
      for (int i = 0; i < n_mine && ok; ++i) {
        const PUnit u = unit_of(a, int(blockIdx.x) + i * int(gridDim.x));
        const PProblem& P = a.pr[u.p];
        const CUtensorMap* wm = u.p ? &w1 : &w0;
        const CUtensorMap* xm = u.p ? &x1 : &x0;
        const uint32_t bytes = uint32_t(kPABytes + P.load_rows * kPKStep * 2);
        for (int ks = 0; ks < a.k_steps; ++ks, ++k) {
          const int st = k % kPStages;
          if (!pwait(s, &s.empty[st], ((k / kPStages) & 1) ^ 1, a.err)) { ok = false; break; }
          unsigned char* A = smem + st * kPStageBytes;
          unsigned char* Bt = A + kPABytes;
          mbar_arrive_expect_tx(&s.full[st], bytes);
          tma_load_2d(A, wm, ks * kPKStep, u.l * P.n_out + u.nt * kPTileN, &s.full[st]);
          if (P.is_4d)
            tma_load_4d(Bt, xm, ks * kPKStep, 0, u.l, u.mt * P.seq_per_unit, &s.full[st]);
          else
            tma_load_3d(Bt, xm, ks * kPKStep, u.l, u.mt * P.seq_per_unit, &s.full[st]);
          ++issued;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int k = 0;
      for (int i = 0; i < n_mine && ok; ++i) {
        const PUnit u = unit_of(a, int(blockIdx.x) + i * int(gridDim.x));
        const PProblem& P = a.pr[u.p];
        const int ab = i & 1;
        if (!pwait(s, &s.acc_empty[ab], ((i >> 1) & 1) ^ 1, a.err)) break;
        tc_fence_after();
        const uint32_t id = idesc_bf16(P.act_rows, false, kPTileN);
        const uint32_t d = tmem + uint32_t(ab * kPMaxAct);
        for (int ks = 0; ks < a.k_steps; ++ks, ++k) {
          const int st = k % kPStages;
          if (!pwait(s, &s.full[st], (k / kPStages) & 1, a.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t A = smem_u32(smem + st * kPStageBytes);
          const uint64_t da = sdesc(A, 16, 1024), db = sdesc(A + kPABytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kPKStep / 16; ++kk)  // K = 16 per MMA: 32 bytes along the row
            mma_bf16(d, da + uint32_t(kk * 2), db + uint32_t(kk * 2), id, (ks > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&s.empty[st]);
        }
        if (ok) mma_commit(&s.acc_full[ab]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int sub = warp & 3;
    const uint32_t trow = tmem + (uint32_t(32 * sub) << 16);
    for (int i = 0; i < n_mine; ++i) {
      const PUnit u = unit_of(a, int(blockIdx.x) + i * int(gridDim.x));
      const PProblem& P = a.pr[u.p];
      const int ab = i & 1;
      if (!__all_sync(0xffffffffu, pwait(s, &s.acc_full[ab], (i >> 1) & 1, a.err))) break;
      tc_fence_after();
      const int n = u.nt * kPTileN + 32 * sub + lane;  // this thread's weight row
      const int seq0 = u.mt * P.seq_per_unit;
      const int seqs = min(P.seq_per_unit, a.b - seq0);
      const int rows = seqs * P.rows_per_seq;  // valid activation rows of the tile
      for (int c0 = 0; c0 < P.act_rows; c0 += 32) {
        float v[32];
        tmem_ld32(trow + uint32_t(ab * kPMaxAct + c0), v);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int m = c0 + j;
          if (m < rows) {
            const int sq = seq0 + m / P.rows_per_seq, r = m % P.rows_per_seq;
            P.y[((int64_t(sq) * a.L + u.l) * P.rows_per_seq + r) * P.n_out + n] = __float2bfloat16_rn(v[j]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&s.acc_empty[ab]);
    }
  }

  __syncthreads();
  if (warp == 0 && lane == 0 && s.abort) {
    // let the copies still in flight land before the shared memory is released
    for (int n = issued > kPStages ? issued - kPStages : 0; n < issued; ++n)
      mbar_wait_bounded(&s.full[n % kPStages], (n / kPStages) & 1, kWaitLimit);
  }
  if (warp == 1 && lane == 0 && s.abort) {
    // and the MMAs issued so far, before TMEM is released
    mma_commit(&s.drain);  // tracks every MMA this thread issued
    mbar_wait_bounded(&s.drain, 0, kWaitLimit);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPTmemCols) : "memory");
  }
}

bool encode_bf16(void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                 CUtensorMap* out) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cuuint32_t(rank), base, dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prologue_supported(const Dev& p) {
  return p.dtype == LS_BF16 && p.hidden % kPKStep == 0 && (p.Hq * p.D) % kPTileN == 0 &&
         (2 * p.Hkv * p.D) % kPTileN == 0 && p.B <= kPMaxAct;
}

cudaError_t launch_prologue(const Dev& p, const void* w_kv, const void* w_q, const void* x, void* bkv, void* q,
                            int sms, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(prologue_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  PArgs a{};
  a.b = p.b;
  a.L = p.L;
  a.k_steps = p.hidden / kPKStep;
  a.err = p.err;
  const cuuint64_t hb = cuuint64_t(p.hidden) * 2;
  // problem 0: block queries, X = x [b][L][B][hidden]
  PProblem& Q = a.pr[0];
  Q.n_out = p.Hq * p.D;
  Q.rows_per_seq = p.B;
  Q.seq_per_unit = kPMaxAct / p.B < p.b ? kPMaxAct / p.B : p.b;
  Q.load_rows = Q.seq_per_unit * p.B;
  Q.act_rows = (Q.load_rows + 15) & ~15;
  Q.m_tiles = (p.b + Q.seq_per_unit - 1) / Q.seq_per_unit;
  Q.n_units = p.L * (Q.n_out / kPTileN) * Q.m_tiles;
  Q.is_4d = 1;
  Q.y = static_cast<__nv_bfloat16*>(q);
  // problem 1: boundary keys/values, X = the state's boundary view [b][L][hidden]
  PProblem& K = a.pr[1];
  K.n_out = 2 * p.Hkv * p.D;
  K.rows_per_seq = 1;
  K.seq_per_unit = p.b < kPMaxAct ? p.b : kPMaxAct;
  K.load_rows = K.seq_per_unit;
  K.act_rows = (K.load_rows + 15) & ~15;
  K.m_tiles = (p.b + K.seq_per_unit - 1) / K.seq_per_unit;
  K.n_units = p.L * (K.n_out / kPTileN) * K.m_tiles;
  K.is_4d = 0;
  K.y = static_cast<__nv_bfloat16*>(bkv);
  a.n_units = Q.n_units + K.n_units;

  CUtensorMap mw0, mx0, mw1, mx1;
  {
    const cuuint64_t dims[2] = {cuuint64_t(p.hidden), cuuint64_t(p.L) * Q.n_out};
    const cuuint64_t str[1] = {hb};
    const cuuint32_t box[2] = {kPKStep, kPTileN};
    if (!encode_bf16(const_cast<void*>(w_q), 2, dims, str, box, &mw0)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[4] = {cuuint64_t(p.hidden), cuuint64_t(p.B), cuuint64_t(p.L), cuuint64_t(p.b)};
    const cuuint64_t str[3] = {hb, hb * p.B, hb * p.B * p.L};
    const cuuint32_t box[4] = {kPKStep, cuuint32_t(p.B), 1, cuuint32_t(Q.seq_per_unit)};
    if (!encode_bf16(const_cast<void*>(x), 4, dims, str, box, &mx0)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {cuuint64_t(p.hidden), cuuint64_t(p.L) * K.n_out};
    const cuuint64_t str[1] = {hb};
    const cuuint32_t box[2] = {kPKStep, kPTileN};
    if (!encode_bf16(const_cast<void*>(w_kv), 2, dims, str, box, &mw1)) return cudaErrorInvalidValue;
  }
  {
    // (rows past the batch in a last, partial tile read as zeros: out of the tensor's bounds)
    const cuuint64_t dims[3] = {cuuint64_t(p.hidden), cuuint64_t(p.L), cuuint64_t(p.b)};
    const cuuint64_t str[2] = {hb, hb * p.L};
    const cuuint32_t box[3] = {kPKStep, 1, cuuint32_t(K.load_rows)};
    if (!encode_bf16(p.boundary, 3, dims, str, box, &mx1)) return cudaErrorInvalidValue;
  }
  const int grid = a.n_units < sms ? a.n_units : sms;
  prologue_kernel<<<grid, kPThreads, kPSmemBytes, stream>>>(a, mw0, mx0, mw1, mx1);
  return cudaGetLastError();
}

}  // namespace ls
