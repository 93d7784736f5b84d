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
// Persistent kernel, 7 warps: warp 0 TMA producer of the weights (a ring of 6 stages of 64
// hidden entries of the unit's 128 weight rows, from HBM), warp 6 TMA producer of the
// activations (3 stages of up to 256 rows, mostly from L2), both 128-byte swizzled; warp 1
// TMEM allocator and MMA issuer (double-buffered accumulator, 2 x 256 columns). Every wait,
// MMA issue and commit of the one MMA-issuing thread takes tens of nanoseconds, so a k-step
// costs it one wait and one commit: both producers' copies of k-step k complete on the
// weight ring's barrier of k (two arrivals), and the release of that barrier's stage also
// frees the activation stage of k (the activation ring, 3 deep, is refilled for k-step k
// once k - 3 is released, which the weight ring's barrier of k - 3 tells). Warps 2-5
// epilogue (one TMEM subpartition each: a thread owns one weight row, its outputs go
// through a shared-memory tile so that whole 256-byte output rows leave as 16-byte
// stores). Units: (problem, layer, 128-row weight tile, activation tile), queries first.
// CTA c runs units c, c + grid, ... whole as long as every CTA has one; the k-steps of the
// units left over (boundary tiles, whose outputs are few) are spread evenly over all CTAs,
// so that every SM streams the same weight bytes, and run first. A piece of such a split
// tile leaves its fp32 partial sums in the state's scratch; the last piece of a tile to
// arrive adds them up in piece order (the same sum whatever the arrival order) and stores
// the tile.
// Launched as the programmatic dependent of the kernel before it on the stream: the weights
// (the drafter's parameters, nearly all of the bytes) stream from the start; the
// activations (the block inputs and the boundary view, which that kernel may write: a
// commit writes the boundary view) are read only after the grid dependency wait. Every
// thread triggers this grid's dependents once it has passed that wait.
// Every wait is bounded.
#include "ls_tc.cuh"

namespace ls {

namespace {

constexpr int kPThreads = 224;                       // 7 warps
constexpr int kPKStep = kProKStep;                   // hidden entries per stage
constexpr int kPTileN = kProTileN;                   // weight rows per unit (MMA M)
constexpr int kPMaxAct = kProMaxAct;                 // activation rows per unit (MMA N)
constexpr int kPAStages = 6;                         // weight ring (read from HBM: deeper)
constexpr int kPBStages = 3;                         // activation ring (read from L2)
constexpr int kPABytes = kPTileN * kPKStep * 2;      // 16 KB
constexpr int kPBBytes = kPMaxAct * kPKStep * 2;     // 32 KB
constexpr int kPOutRows = 128;                       // activation rows per epilogue pass
constexpr int kPOutBytes = kPOutRows * kPTileN * 2;  // 32 KB: [128 rows][128 weight rows] bf16
constexpr int kPSmemBytes = kPAStages * kPABytes + kPBStages * kPBBytes + kPOutBytes + 1024;
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
  int32_t n_full;     // units [0, n_full) run whole, round robin over the CTAs
  int32_t rem_steps;  // k-steps of the split units [n_full, n_units) (all boundary tiles), 0 if none
  float* part;        // [slot][128][pr[1].act_rows] partial sums of the split tiles' pieces
  int32_t* count;     // [unit - n_full] arrivals of a split tile's pieces (zero between calls)
  int32_t* err;
};

struct PBars {
  uint64_t afull[kPAStages], aempty[kPAStages];  // per k-step k: stage k mod kPAStages of
                                                 // both rings full (2 arrivals) / released
  uint64_t acc_full[2], acc_empty[2];
  uint64_t out_full, out_free;  // epilogue pass: staged by all 128 threads / copied out
  uint64_t drain;               // after an abort: the MMAs issued so far have completed
  uint64_t epi;                 // the 128 epilogue threads meet (split tiles' arrivals)
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t last;                // the epilogue's piece was its tile's last to arrive
  int32_t issued[2];            // k-steps each producer arrived for (weights, activations)
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

// This CTA's work: pieces of the split units first (a contiguous range of their flattened
// k-steps, [g0, g1) = [c T / grid, (c + 1) T / grid)), then its whole units. With the
// pieces first, the sum of a split tile (by its last piece to arrive) runs in the epilogue
// warps while the CTA's whole units stream, instead of after them.
struct PWork {
  int n_pieces, n_items;
  int64_t g0, g1;
};

struct PItem {
  int u;       // unit
  int k0, k1;  // its k-steps [k0, k1)
  int slot;    // -1: the whole unit; else the piece's partial-sum slot
  int r;       // split unit index (u - n_full)
};

__device__ inline int64_t range_begin(int c, int64_t T, int grid) { return int64_t(c) * T / grid; }

// the CTA whose range holds split k-step g: the largest c with c T / grid <= g (rounded down)
__device__ inline int range_cta(int64_t g, int64_t T, int grid) { return int(((g + 1) * grid + T - 1) / T) - 1; }

__device__ inline PWork work_of(const PArgs& a) {
  PWork w;
  const int c = int(blockIdx.x), G = int(gridDim.x);
  const int n_whole = c < a.n_full ? (a.n_full - 1 - c) / G + 1 : 0;
  w.g0 = range_begin(c, a.rem_steps, G);
  w.g1 = range_begin(c + 1, a.rem_steps, G);
  w.n_pieces = w.g1 > w.g0 ? int((w.g1 - 1) / a.k_steps - w.g0 / a.k_steps + 1) : 0;
  w.n_items = w.n_pieces + n_whole;
  return w;
}

__device__ inline PItem item_of(const PArgs& a, const PWork& w, int i) {
  PItem it;
  if (i >= w.n_pieces) {
    it.u = int(blockIdx.x) + (i - w.n_pieces) * int(gridDim.x);
    it.k0 = 0;
    it.k1 = a.k_steps;
    it.slot = -1;
    it.r = -1;
    return it;
  }
  it.r = int(w.g0 / a.k_steps) + i;
  const int64_t lo = int64_t(it.r) * a.k_steps;
  it.u = a.n_full + it.r;
  it.k0 = int((w.g0 > lo ? w.g0 : lo) - lo);
  it.k1 = int((w.g1 < lo + a.k_steps ? w.g1 : lo + a.k_steps) - lo);
  // (CTA, split unit) pairs are ordered the same way in both: c + r is unique per piece
  it.slot = int(blockIdx.x) + it.r;
  return it;
}

// uses of stage st among the first n k-steps of a ring of nst stages
__device__ inline int stage_uses(int n, int st, int nst) { return n > st ? (n - 1 - st) / nst + 1 : 0; }

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
  unsigned char* a_ring = smem;                              // [kPAStages][16 KB]
  unsigned char* b_ring = a_ring + kPAStages * kPABytes;     // [kPBStages][32 KB]
  unsigned char* out_st = b_ring + kPBStages * kPBBytes;     // [128][128] bf16
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PWork w = work_of(a);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPAStages; ++i) { mbar_init(&s.afull[i], 2); mbar_init(&s.aempty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&s.acc_full[i], 1); mbar_init(&s.acc_empty[i], 128); }
    mbar_init(&s.out_full, 128);
    mbar_init(&s.out_free, 128);
    mbar_init(&s.drain, 1);
    mbar_init(&s.epi, 128);
    s.abort = 0;
    s.issued[0] = s.issued[1] = 0;
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
  if (warp != 0) {  // the weight producer waits once its first ring of weights is on its way
    grid_dependency_wait();
    allow_dependent_launch();
  }

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------ TMA producers
    // warp 0: the weights (A) of every k-step; warp 6: the activations (B)
    bool waited = warp != 0;
    if (lane == 0) {
      const bool is_a = warp == 0;
      const int nst = is_a ? kPAStages : kPBStages;
      prefetch_map(is_a ? &w0 : &x0);
      prefetch_map(is_a ? &w1 : &x1);
      const uint64_t pol = is_a ? l2_evict_first() : l2_evict_last();
      bool ok = true;
      int k = 0;
      for (int i = 0; i < w.n_items && ok; ++i) {
        const PItem it = item_of(a, w, i);
        const PUnit u = unit_of(a, it.u);
        const PProblem& P = a.pr[u.p];
        const CUtensorMap* m = is_a ? (u.p ? &w1 : &w0) : (u.p ? &x1 : &x0);
        const uint32_t bytes = is_a ? uint32_t(kPABytes) : uint32_t(P.load_rows * kPKStep * 2);
        // the weights are read once: they must not push the activations (read again by
        // every weight tile of the layer) out of L2
        for (int ks = it.k0; ks < it.k1; ++ks, ++k) {
          const int st = k % nst;          // this ring's stage
          uint64_t* full = &s.afull[k % kPAStages];  // the k-step's barrier
          if (k == nst && !waited) {  // (the first ring's weights are in flight)
            grid_dependency_wait();
            allow_dependent_launch();
            waited = true;
          }
          // the stage is free once the MMAs of the k-step that used it before have completed
          // (k - nst); the MMAs of a k-step complete in order, and the one wait before for
          // the same barrier covered its previous phase, so the parity names this phase
          const int prev = k - nst;
          if (prev >= 0 && !pwait(s, &s.aempty[prev % kPAStages], uint32_t(prev / kPAStages) & 1, a.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full, bytes);
          if (is_a)
            tma_load_2d_hint(a_ring + st * kPABytes, m, ks * kPKStep, u.l * P.n_out + u.nt * kPTileN, full, pol);
          else if (P.is_4d)
            tma_load_4d_hint(b_ring + st * kPBBytes, m, ks * kPKStep, 0, u.l, u.mt * P.seq_per_unit, full, pol);
          else
            tma_load_3d_hint(b_ring + st * kPBBytes, m, ks * kPKStep, u.l, u.mt * P.seq_per_unit, full, pol);
        }
      }
      s.issued[is_a ? 0 : 1] = k;
    }
    if (!waited) {  // (every thread of the CTA passes the wait before it triggers)
      grid_dependency_wait();
      allow_dependent_launch();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int k = 0;
      for (int i = 0; i < w.n_items && ok; ++i) {
        const PItem it = item_of(a, w, i);
        const PUnit u = unit_of(a, it.u);
        const PProblem& P = a.pr[u.p];
        const int ab = i & 1;
        if (!pwait(s, &s.acc_empty[ab], ((i >> 1) & 1) ^ 1, a.err)) break;
        tc_fence_after();
        const uint32_t id = idesc_bf16(P.act_rows, false, kPTileN);
        const uint32_t d = tmem + uint32_t(ab * kPMaxAct);
        for (int ks = it.k0; ks < it.k1; ++ks, ++k) {
          const int sa = k % kPAStages, sb = k % kPBStages;
          if (!pwait(s, &s.afull[sa], (k / kPAStages) & 1, a.err)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = sdesc(smem_u32(a_ring + sa * kPABytes), 16, 1024);
          const uint64_t db = sdesc(smem_u32(b_ring + sb * kPBBytes), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kPKStep / 16; ++kk)  // K = 16 per MMA: 32 bytes along the row
            mma_bf16(d, da + uint32_t(kk * 2), db + uint32_t(kk * 2), id, (ks > it.k0 || kk > 0) ? 1u : 0u);
          mma_commit(&s.aempty[sa]);  // frees both stages of the k-step
        }
        if (ok) mma_commit(&s.acc_full[ab]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    // Per 128 activation rows: each thread writes its weight row's outputs (a column of the
    // staging tile [row][128 weight rows]), then all 128 threads copy the tile's valid rows
    // out as 16-byte pieces of 256-byte output rows. fetch(col, v) gives the thread's 32
    // accumulator values of activation rows col .. col + 31 (TMEM, or summed partials).
    const int sub = warp & 3;
    const int ecol = 32 * sub + lane;  // this thread's weight row within the unit
    const int etid = threadIdx.x - 64;  // 0..127
    const uint32_t trow = tmem + (uint32_t(32 * sub) << 16);
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(out_st);
    int pass = 0;  // epilogue passes so far (phases of out_full / out_free)
    int meets = 0;  // phases of `epi` so far
    bool ok = true;
    // all 128 epilogue threads meet here (bounded: a thread that gave up makes the rest give up)
    auto epi_meet = [&]() -> bool {
      mbar_arrive(&s.epi);
      return __all_sync(0xffffffffu, pwait(s, &s.epi, uint32_t(meets++) & 1, a.err));
    };
    auto store_tile = [&](const PUnit& u, const PProblem& P, auto&& fetch) -> bool {
      const int seq0 = u.mt * P.seq_per_unit;
      const int rows = min(P.seq_per_unit, a.b - seq0) * P.rows_per_seq;  // valid activation rows
      for (int r0 = 0; r0 < rows; r0 += kPOutRows, ++pass) {
        // the staging tile is free once every thread has copied the previous pass out
        if (pass > 0 && !__all_sync(0xffffffffu, pwait(s, &s.out_free, (pass - 1) & 1, a.err))) return false;
        const int nr = min(kPOutRows, P.act_rows - r0);
        for (int c0 = 0; c0 < nr; c0 += 32) {
          float v[32];
          fetch(r0 + c0, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) stage[(c0 + j) * kPTileN + ecol] = __float2bfloat16_rn(v[j]);
        }
        mbar_arrive(&s.out_full);
        if (!__all_sync(0xffffffffu, pwait(s, &s.out_full, pass & 1, a.err))) return false;
        const int vr = min(kPOutRows, rows - r0);
        for (int c = etid; c < vr * 16; c += 128) {  // 16 pieces of 16 bytes per row
          const int m = r0 + (c >> 4);
          const int sq = seq0 + m / P.rows_per_seq, r = m % P.rows_per_seq;
          uint4* dst = reinterpret_cast<uint4*>(P.y + ((int64_t(sq) * a.L + u.l) * P.rows_per_seq + r) * P.n_out +
                                                u.nt * kPTileN) + (c & 15);
          *dst = reinterpret_cast<const uint4*>(stage + (c >> 4) * kPTileN)[c & 15];
        }
        mbar_arrive(&s.out_free);
      }
      return true;
    };
    for (int i = 0; i < w.n_items && ok; ++i) {
      const PItem it = item_of(a, w, i);
      const PUnit u = unit_of(a, it.u);
      const PProblem& P = a.pr[u.p];
      const int ab = i & 1;
      if (!__all_sync(0xffffffffu, pwait(s, &s.acc_full[ab], (i >> 1) & 1, a.err))) break;
      tc_fence_after();
      if (it.slot < 0) {
        ok = store_tile(u, P, [&](int col, float (&v)[32]) { tmem_ld32(trow + uint32_t(ab * kPMaxAct + col), v); });
        tc_fence_before();
        mbar_arrive(&s.acc_empty[ab]);
        continue;
      }
      // a piece of a split tile: its partial sums (this thread's weight row, all activation
      // rows) go to its slot, and the accumulator is released at once
      const int na = P.act_rows;  // a multiple of 16
      float* mine = a.part + (int64_t(it.slot) * kPTileN + ecol) * na;
      for (int c0 = 0; c0 < na; c0 += 32) {
        float v[32];
        tmem_ld32(trow + uint32_t(ab * kPMaxAct + c0), v);
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          if (c0 + j < na) *reinterpret_cast<float4*>(mine + c0 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      }
      tc_fence_before();
      mbar_arrive(&s.acc_empty[ab]);
      __threadfence();  // this thread's partials are visible before the arrival below
      if (!epi_meet()) { ok = false; break; }
      const int64_t T = a.rem_steps;
      const int G = int(gridDim.x);
      const int c_first = range_cta(int64_t(it.r) * a.k_steps, T, G);
      const int c_last = range_cta(int64_t(it.r + 1) * a.k_steps - 1, T, G);
      if (etid == 0) s.last = atomicAdd(a.count + it.r, 1) == c_last - c_first ? 1u : 0u;
      if (!epi_meet()) { ok = false; break; }
      if (!s.last) continue;
      __threadfence();  // every piece's partials are visible from here on
      ok = store_tile(u, P, [&](int col, float (&v)[32]) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
        for (int c = c_first; c <= c_last; ++c) {  // slot order: the same sum for every arrival order
          const float* src = a.part + (int64_t(c + it.r) * kPTileN + ecol) * na + col;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            if (col + j < na) {
              const float4 x = __ldcg(reinterpret_cast<const float4*>(src + j));
              v[j] += x.x; v[j + 1] += x.y; v[j + 2] += x.z; v[j + 3] += x.w;
            }
          }
        }
      });
      if (etid == 0) a.count[it.r] = 0;  // ready for the next call
    }
  }

  __syncthreads();
  if (warp == 0 && lane == 0 && s.abort) {
    // let the copies still in flight land before the shared memory is released: a k-step
    // barrier that only one producer arrived for (the other gave up first; the producers
    // are at most a ring apart, so by one use of a barrier) gets the other's arrival, then
    // each barrier's last phase completes once its copies have landed
    for (int st = 0; st < kPAStages; ++st) {
      const int na = stage_uses(s.issued[0], st, kPAStages), nb = stage_uses(s.issued[1], st, kPAStages);
      if (na != nb) mbar_arrive(&s.afull[st]);
      const int n = na > nb ? na : nb;
      if (n > 0) mbar_wait_bounded(&s.afull[st], uint32_t(n - 1) & 1, kWaitLimit);
    }
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

bool prologue_supported(const Dev& p) { return prologue_shapes_ok(p.dtype, p.hidden, p.Hq, p.Hkv, p.D, p.B); }

cudaError_t launch_prologue(const Dev& p, const void* w_kv, const void* w_q, const void* x, void* bkv, void* q,
                            int sms, cudaStream_t stream) {
  // per launch: the attribute belongs to the current device's copy of the kernel
  cudaError_t e = cudaFuncSetAttribute(prologue_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmemBytes);
  if (e != cudaSuccess) return e;
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
  int grid = sms < kProMaxGrid ? sms : kProMaxGrid;
  if (a.n_units < grid) grid = a.n_units;
  // units left over after whole waves: split their k-steps over every CTA when they are all
  // boundary tiles (their partial sums fit the state's scratch: 128 x K.act_rows fp32 each)
  // and there are at least as many k-steps as CTAs (then every CTA's range is non-empty, so
  // a tile's pieces are those of the CTAs from the one holding its first k-step to the one
  // holding its last; with fewer, the CTAs between could hold none and the tile's arrival
  // count would never be reached)
  const int rem = a.n_units % grid;
  const bool split = rem > 0 && rem <= K.n_units && K.act_rows == prologue_boundary_rows(p.b) &&
                     int64_t(rem) * a.k_steps >= grid;
  a.n_full = split ? a.n_units - rem : a.n_units;
  a.rem_steps = split ? rem * a.k_steps : 0;
  a.part = p.pro_part;
  a.count = p.pro_count;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = kPSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prologue_kernel, a, mw0, mx0, mw1, mx1);
}

}  // namespace ls
