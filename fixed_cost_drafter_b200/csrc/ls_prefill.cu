// Summary initialisation over the full prefix at target prefill: LongSpark paper page,
// Figure 3 caption ("initialized over the full prefix during target prefill").
//
// Pass 1 (prefill_units_kernel, persistent, one CTA per SM): the work items are units
// of U prefix rows of one (sequence, layer); U is the largest scale <= 512. A producer
// warp streams each unit's K and V rows (all KV heads of a row are contiguous; from a
// dense input, or in place from the target's paged cache, one copy per page run) through
// the TMA engine into a ring of shared-memory stages (cp.async.bulk + mbarrier
// transaction counts; the consumers release a stage through an "empty" mbarrier, no
// block-wide barrier); every consumer thread owns one 16-byte column vector and keeps
// one fp32 sum per scale <= U, adding rows in runs between segment closes. When a
// segment of scale s_k closes, its sum is added into the next scale's sum (a tree,
// not a long serial chain) and, if the segment is among the `slots` most recent ones of
// the final prefix, its mean is written. A closed unit's sum goes to the workspace.
// The last W prefix rows are copied into the ring window on the way through.
// Pass 2 (prefill_finalize_kernel): per (sequence, layer, column block) the unit sums
// are combined the same way into the segments of the scales > U, the partial sums, the
// global sum (accumulated across chunk calls), the mean rows and the counters.
#include <mutex>

#include "ls_common.cuh"

namespace ls {

struct PrefillArgs {
  const char* k;
  const char* v;
  int64_t plane_stride, row_stride;  // elements
  const int64_t* prefix_len;
  int64_t row_begin, row_end;
  float* ws;        // [b*L][n_units][2*Hkv*D] unit sums
  int32_t n_units;  // units per (sequence, layer) in this chunk
  int32_t U;        // unit rows (a scale)
  int32_t kU;       // scales 0..kU-1 are <= U (scale kU-1 == U)
  int32_t G;        // rows per stage
  int32_t n_items;  // b * L * n_units
};

constexpr int kPrefillThreads = 256;                 // consumer threads
constexpr int kPrefillBlock = kPrefillThreads + 32;  // + one producer warp
constexpr int kPrefillStages = 3;

__device__ inline int64_t clamp_prefix(const PrefillArgs& a, const Dev&, int b) {
  int64_t P = a.prefix_len[b];
  return P < 0 ? 0 : P;
}

// rows [r0, r1) of item `it` inside this chunk (empty when r1 <= r0)
__device__ inline void item_rows(const PrefillArgs& a, const Dev& p, int it, int& bl, int& u,
                                 int64_t& r0, int64_t& r1) {
  bl = it / a.n_units;
  u = it - bl * a.n_units;
  const int b = bl / p.L;
  const int64_t end = min(a.row_end, clamp_prefix(a, p, b));
  r0 = a.row_begin + int64_t(u) * a.U;
  r1 = min(r0 + a.U, end);
}

// Cursor over the flattened (item, row group) stage sequence of one CTA.
struct Cursor {
  int j;        // item ordinal within this CTA (item = blockIdx.x + j * gridDim.x)
  int grp;      // row group within the item
  bool valid;
};

__device__ inline void cursor_settle(const PrefillArgs& a, const Dev& p, Cursor& c) {
  // move forward to the first item with rows left at group c.grp
  while (true) {
    const int it = blockIdx.x + c.j * gridDim.x;
    if (it >= a.n_items) { c.valid = false; return; }
    int bl, u; int64_t r0, r1;
    item_rows(a, p, it, bl, u, r0, r1);
    if (r1 > r0 + int64_t(c.grp) * a.G) { c.valid = true; return; }
    c.j += 1; c.grp = 0;
  }
}
__device__ inline void cursor_next(const PrefillArgs& a, const Dev& p, Cursor& c) {
  c.grp += 1;
  cursor_settle(a, p, c);
}

// Where the prefix rows come from: the dense [b*L planes][rows][Hkv][D] input (a.k, a.v)
// or the target's paged KV cache read in place.
struct DensePrefix {};

// Issues the bulk copies of rows [g0, g0 + nrows) of tensor t (0 = K, 1 = V) of (sequence,
// layer) bl into dst (rows of rowBytes bytes, back to back), completing on `bar`.
template <typename T>
__device__ inline void issue_prefix_rows(const Dev&, const PrefillArgs& a, const DensePrefix&, int t, int bl,
                                         int64_t g0, int nrows, char* dst, int rowBytes, uint64_t* bar) {
  const char* base = (t == 0 ? a.k : a.v) +
                     (int64_t(bl) * a.plane_stride + (g0 - a.row_begin) * a.row_stride) * int64_t(sizeof(T));
  if (a.row_stride * int64_t(sizeof(T)) == rowBytes) {
    bulk_g2s(dst, base, uint32_t(nrows * rowBytes), bar);
  } else {
    for (int r = 0; r < nrows; ++r)
      bulk_g2s(dst + r * rowBytes, base + int64_t(r) * a.row_stride * int64_t(sizeof(T)), uint32_t(rowBytes), bar);
  }
}

// Paged: one copy per run of rows inside a page (per row when the slots are not packed).
// The producer loads a stage's block-table entries one stage ahead (PrefixLookup: the loads
// are issued, their values used an iteration later) and turns them into the copies' source
// addresses (PrefixPlan) before it waits for the stage's buffer, so the entries' latency
// overlaps the stage before instead of delaying the refill.
struct PrefixLookup {
  static constexpr int kMaxRuns = 2;  // a stage of G rows spans at most 2 pages when page_size >= G
  int32_t entry[kMaxRuns];  // the runs' block-table entries (loads in flight)
  int off[kMaxRuns], r0[kMaxRuns], n[kMaxRuns], nrun;
  bool ok;  // false: the stage needs more runs, issue_prefix_rows looks it up after the wait
};
struct PrefixPlan {
  static constexpr int kMaxRuns = PrefixLookup::kMaxRuns;
  const char* src[2][kMaxRuns];
  int r0[kMaxRuns], n[kMaxRuns], nrun;
  bool ok;
};

__device__ inline int page_offset(int64_t pos, int ps) {
  if ((ps & (ps - 1)) == 0) return int(pos & (ps - 1));
  if (pos < (int64_t(1) << 32)) return int(uint32_t(pos) % uint32_t(ps));
  return int(pos % ps);
}

template <typename T>
__device__ inline void lookup_prefix_rows(const Dev&, const DensePrefix&, int, int64_t, int, PrefixLookup& lk) {
  lk.ok = false;  // dense: addresses are plain arithmetic, nothing to look up
}

template <typename T>
__device__ inline void lookup_prefix_rows(const Dev& p, const ls_paged_kv& kv, int bl, int64_t g0, int nrows,
                                          PrefixLookup& lk) {
  const int b = bl / p.L;
  int r = 0;
  lk.nrun = 0;
  // (fixed trip count: the lookup stays in registers)
#pragma unroll
  for (int k = 0; k < PrefixLookup::kMaxRuns; ++k) {
    lk.entry[k] = -1;
    lk.off[k] = 0;
    lk.r0[k] = r;
    lk.n[k] = 0;
    if (r < nrows) {
      const int64_t pos = g0 + r;
      const int64_t pi = paged_index(kv, pos, lk.off[k]);
      lk.entry[k] = paged_entry(kv, b, pi);
      lk.n[k] = min(nrows - r, kv.page_size - lk.off[k]);
      lk.nrun = k + 1;
      r += lk.n[k];
    }
  }
  lk.ok = r >= nrows;
}

template <typename T>
__device__ inline void plan_prefix_rows(const Dev&, const DensePrefix&, int, const PrefixLookup&, PrefixPlan& pl) {
  pl.ok = false;
}

template <typename T>
__device__ inline void plan_prefix_rows(const Dev& p, const ls_paged_kv& kv, int bl, const PrefixLookup& lk,
                                        PrefixPlan& pl) {
  const int l = bl - (bl / p.L) * p.L;
  pl.ok = lk.ok;
  pl.nrun = lk.nrun;
#pragma unroll
  for (int k = 0; k < PrefixPlan::kMaxRuns; ++k) {
    pl.r0[k] = lk.r0[k];
    pl.n[k] = lk.n[k];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const char* base = static_cast<const char*>(t == 0 ? kv.k_layers[l] : kv.v_layers[l]);
      pl.src[t][k] = k < lk.nrun ? paged_at(kv, base, lk.entry[k], lk.off[k], int(sizeof(T)), p.err) : nullptr;
    }
  }
}

template <typename T>
__device__ inline void issue_plan(const ls_paged_kv& kv, const PrefixPlan& pl, int t, char* dst, int rowBytes,
                                  uint64_t* bar) {
  const bool packed = kv.slot_stride * int64_t(sizeof(T)) == rowBytes;
#pragma unroll
  for (int k = 0; k < PrefixPlan::kMaxRuns; ++k) {
    if (k >= pl.nrun) break;
    if (packed) {
      bulk_g2s(dst + pl.r0[k] * rowBytes, pl.src[t][k], uint32_t(pl.n[k] * rowBytes), bar);
    } else {
      for (int i = 0; i < pl.n[k]; ++i)
        bulk_g2s(dst + (pl.r0[k] + i) * rowBytes, pl.src[t][k] + int64_t(i) * kv.slot_stride * int64_t(sizeof(T)),
                 uint32_t(rowBytes), bar);
    }
  }
}
template <typename T>
__device__ inline void issue_plan(const DensePrefix&, const PrefixPlan&, int, char*, int, uint64_t*) {}

// Paged, unplanned (a stage spanning more than 2 pages): lookups after the wait.
template <typename T>
__device__ inline void issue_prefix_rows(const Dev& p, const PrefillArgs&, const ls_paged_kv& kv, int t, int bl,
                                         int64_t g0, int nrows, char* dst, int rowBytes, uint64_t* bar) {
  const int b = bl / p.L, l = bl - b * p.L;
  const char* base = static_cast<const char*>(t == 0 ? kv.k_layers[l] : kv.v_layers[l]);
  const bool packed = kv.slot_stride * int64_t(sizeof(T)) == rowBytes;
  int r = 0;
  while (r < nrows) {
    const int64_t pos = g0 + r;
    const int run = min(nrows - r, kv.page_size - page_offset(pos, kv.page_size));
    const char* src = paged_row(kv, base, b, pos, int(sizeof(T)), p.err);
    if (packed) {
      bulk_g2s(dst + r * rowBytes, src, uint32_t(run * rowBytes), bar);
    } else {
      for (int i = 0; i < run; ++i)
        bulk_g2s(dst + (r + i) * rowBytes, src + int64_t(i) * kv.slot_stride * int64_t(sizeof(T)),
                 uint32_t(rowBytes), bar);
    }
    r += run;
  }
}

template <typename T, int CVT, typename Src>
__global__ void __launch_bounds__(kPrefillBlock, 1)
prefill_units_kernel(Dev p, PrefillArgs a, const Src src) {
  using E = Elem<T>;
  constexpr int VEC = E::kVec;
  extern __shared__ __align__(128) char smem[];
  __shared__ uint64_t full[kPrefillStages], empty[kPrefillStages];
  __shared__ uint32_t abort_flag;

  const int rowElems = p.Hkv * p.D;
  const int rowBytes = rowElems * int(sizeof(T));
  const int stageBytes = 2 * a.G * rowBytes;
  const int ncv = 2 * rowElems / VEC;  // column vectors of K then V
  const int cvPerRow = rowElems / VEC;
  const int tid = threadIdx.x;

  if (tid == 0) {
    for (int s = 0; s < kPrefillStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kPrefillThreads); }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // bounded wait that also gives up once another thread has given up
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
#pragma unroll 1
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
      if (mbar_try_wait(bar, parity)) return true;
      if ((i & 1023) == 1023 && *reinterpret_cast<volatile uint32_t*>(&abort_flag)) return false;
    }
    set_err(p.err, LS_DEVERR_WAIT_TIMEOUT);
    *reinterpret_cast<volatile uint32_t*>(&abort_flag) = 1;
    return false;
  };

  if (tid >= kPrefillThreads) {
    // ------------------------------------------------------------ producer (one lane)
    // stage n goes into buffer n % kPrefillStages once the consumers released it
    if (tid == kPrefillThreads) {
      Cursor prod{0, 0, false};
      cursor_settle(a, p, prod);
      int n = 0;
      int last_issue[kPrefillStages];
      for (int s = 0; s < kPrefillStages; ++s) last_issue[s] = -1;
      // the rows of the stage at cursor c
      auto stage_rows = [&](const Cursor& c, int& bl, int64_t& g0, int& nrows) {
        const int it = blockIdx.x + c.j * gridDim.x;
        int u; int64_t r0, r1;
        item_rows(a, p, it, bl, u, r0, r1);
        g0 = r0 + int64_t(c.grp) * a.G;
        nrows = int(min(int64_t(a.G), r1 - g0));
      };
      int bl = 0, nrows = 0;
      int64_t g0 = 0;
      PrefixLookup look;
      if (prod.valid) {
        stage_rows(prod, bl, g0, nrows);
        lookup_prefix_rows<T>(p, src, bl, g0, nrows, look);
      }
      for (; prod.valid; ++n) {
        const int buf = n % kPrefillStages;
        // the next stage's page lookups go out now; this stage's (loaded one stage ago)
        // become its copies' addresses before waiting for the buffer
        Cursor nx = prod;
        cursor_next(a, p, nx);
        int nbl = 0, nnrows = 0;
        int64_t ng0 = 0;
        PrefixLookup nlook;
        nlook.ok = false;
        if (nx.valid) {
          stage_rows(nx, nbl, ng0, nnrows);
          lookup_prefix_rows<T>(p, src, nbl, ng0, nnrows, nlook);
        }
        PrefixPlan plan;
        plan_prefix_rows<T>(p, src, bl, look, plan);
        if (!wait(&empty[buf], ((n / kPrefillStages) & 1) ^ 1)) break;
        fence_proxy_async_smem();  // the consumers' reads of the buffer come before its refill
        char* dst = smem + buf * stageBytes;
        mbar_arrive_expect_tx(&full[buf], uint32_t(2 * nrows * rowBytes));
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (plan.ok)
            issue_plan<T>(src, plan, t, dst + t * a.G * rowBytes, rowBytes, &full[buf]);
          else
            issue_prefix_rows<T>(p, a, src, t, bl, g0, nrows, dst + t * a.G * rowBytes, rowBytes, &full[buf]);
        }
        last_issue[buf] = n;
        prod = nx;
        bl = nbl;
        g0 = ng0;
        nrows = nnrows;
        look = nlook;
      }
      if (*reinterpret_cast<volatile uint32_t*>(&abort_flag)) {
        // let every copy still in flight land before the CTA's shared memory goes away
        for (int s = 0; s < kPrefillStages; ++s)
          if (last_issue[s] >= 0)
            mbar_wait_bounded(&full[s], uint32_t((last_issue[s] / kPrefillStages) & 1), kWaitLimit);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    // this thread's column vectors (fixed for the whole kernel): K (0) or V (1), head,
    // element offset in the head, byte offset in the row
    bool col_ok[CVT];
    int col_t[CVT], col_h[CVT], col_d0[CVT], col_byte[CVT], col_kv[CVT];
#pragma unroll
    for (int q = 0; q < CVT; ++q) {
      const int cv = tid + q * kPrefillThreads;
      col_ok[q] = cv < ncv;
      const int t = cv / cvPerRow, e0 = (cv - t * cvPerRow) * VEC;
      col_t[q] = t;
      col_h[q] = e0 / p.D;
      col_d0[q] = e0 - col_h[q] * p.D;
      col_byte[q] = e0 * int(sizeof(T));
      col_kv[q] = col_h[q] * 2 + t;  // (head, K|V) plane of the (sequence, layer)
    }
    Cursor cons{0, 0, false};
    cursor_settle(a, p, cons);
    int consumed = 0;
    float acc[CVT][kMaxScales + 1][VEC];
    int cnt[kMaxScales];  // rows (k = 0) or closes of scale k-1 until scale k closes
    int cur_item = -1;

    while (cons.valid) {
      const int it = blockIdx.x + cons.j * gridDim.x;
      int bl, u; int64_t r0, r1;
      item_rows(a, p, it, bl, u, r0, r1);
      const int b = bl / p.L;
      const int64_t P = clamp_prefix(a, p, b);
      if (it != cur_item) {  // new item: all sums start empty (r0 is a multiple of U)
        cur_item = it;
#pragma unroll
        for (int q = 0; q < CVT; ++q)
#pragma unroll
          for (int k = 0; k <= kMaxScales; ++k)
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[q][k][e] = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxScales; ++k)
          cnt[k] = k >= a.kU ? 0 : (k == 0 ? p.scales[0] : p.scales[k] / p.scales[k - 1]);
      }
      const int64_t g0 = r0 + int64_t(cons.grp) * a.G;
      const int nrows = int(min(int64_t(a.G), r1 - g0));
      const int buf = consumed % kPrefillStages;
      if (!wait(&full[buf], uint32_t((consumed / kPrefillStages) & 1))) break;

      const char* st = smem + buf * stageBytes;
      // rows >= wfirst of this stage are among the prefix's last W: ring slot pos mod W
      const int64_t wf = P - p.W > g0 ? P - p.W - g0 : 0;
      const int wfirst = wf < nrows ? int(wf) : nrows;
      int wslot = wfirst < nrows ? int((g0 + wfirst) % p.W) : 0;
      int r = 0;
      while (r < nrows) {
        // rows up to and including the next close of the smallest scale
        const int run = nrows - r < cnt[0] ? nrows - r : cnt[0];
        const int rend = r + run;
        if (rend <= wfirst) {  // no ring-window row in this run
#pragma unroll 4
          for (; r < rend; ++r) {
#pragma unroll
            for (int q = 0; q < CVT; ++q) {
              if (!col_ok[q]) continue;
              const uint4 raw = *reinterpret_cast<const uint4*>(st + (col_t[q] * a.G + r) * rowBytes + col_byte[q]);
              float f[VEC];
              E::to_f32(raw, f);
#pragma unroll
              for (int e = 0; e < VEC; ++e) acc[q][0][e] += f[e];
            }
          }
        } else {
          for (; r < rend; ++r) {
#pragma unroll
            for (int q = 0; q < CVT; ++q) {
              if (!col_ok[q]) continue;
              const uint4 raw = *reinterpret_cast<const uint4*>(st + (col_t[q] * a.G + r) * rowBytes + col_byte[q]);
              float f[VEC];
              E::to_f32(raw, f);
#pragma unroll
              for (int e = 0; e < VEC; ++e) acc[q][0][e] += f[e];
              if (r >= wfirst) {
                T* kvt = reinterpret_cast<T*>(p.kv) + (int64_t(bl) * p.Hkv * 2 + col_kv[q]) * int64_t(p.R) * p.D;
                *reinterpret_cast<uint4*>(kvt + int64_t(wslot) * p.D + col_d0[q]) = raw;
              }
            }
            if (r >= wfirst && ++wslot == p.W) wslot = 0;
          }
        }
        cnt[0] -= run;
        if (cnt[0] != 0) break;  // r == nrows: no close in the rest of the stage
        // segment closes at row rend - 1, smallest scale first; a closed scale feeds the next
        const int64_t pos = g0 + rend - 1;
#pragma unroll
        for (int k = 0; k < kMaxScales; ++k) {
          if (k >= a.kU) break;
          if (k > 0 && --cnt[k] != 0) break;  // level k counts closes of level k-1
          cnt[k] = k == 0 ? p.scales[0] : p.scales[k] / p.scales[k - 1];
          const int s = p.scales[k];
          const int64_t j = pos / s;  // segment that just closed
          const bool keep = j >= P / s - p.slots;
#pragma unroll
          for (int q = 0; q < CVT; ++q) {
            if (!col_ok[q]) continue;
            const int cv = tid + q * kPrefillThreads;
            const int64_t tile = int64_t(bl) * p.Hkv + col_h[q];
            if (keep) {
              float m[VEC];
#pragma unroll
              for (int e = 0; e < VEC; ++e) m[e] = acc[q][k][e] / float(s);
              const int slot = int(j % p.slots);
              float* sg = p.seg + (((tile * p.nsc + k) * p.slots + slot) * 2 + col_t[q]) * p.D + col_d0[q];
#pragma unroll
              for (int e = 0; e < VEC; e += 4)
                *reinterpret_cast<float4*>(sg + e) = make_float4(m[e], m[e + 1], m[e + 2], m[e + 3]);
              T* kvt = reinterpret_cast<T*>(p.kv) + (tile * 2 + col_t[q]) * int64_t(p.R) * p.D;
              *reinterpret_cast<uint4*>(kvt + (int64_t(p.W) + k * (p.slots + 1) + slot) * p.D + col_d0[q]) =
                  E::from_f32(m);
            }
            if (k + 1 < a.kU) {
#pragma unroll
              for (int e = 0; e < VEC; ++e) { acc[q][k + 1][e] += acc[q][k][e]; acc[q][k][e] = 0.f; }
            } else {  // the unit closed: its sum goes to the workspace
              float* w = a.ws + (int64_t(bl) * a.n_units + u) * (2 * rowElems) + int64_t(cv) * VEC;
#pragma unroll
              for (int e = 0; e < VEC; e += 4)
                *reinterpret_cast<float4*>(w + e) =
                    make_float4(acc[q][k][e], acc[q][k][e + 1], acc[q][k][e + 2], acc[q][k][e + 3]);
#pragma unroll
              for (int e = 0; e < VEC; ++e) acc[q][k][e] = 0.f;
            }
          }
        }
      }
      mbar_arrive(&empty[buf]);  // this thread's reads of the stage are done

      if (g0 + nrows == r1) {  // the item ends with this stage
        const bool unit_closed = r1 - r0 == a.U;
#pragma unroll
        for (int q = 0; q < CVT; ++q) {
          if (!col_ok[q]) continue;
          const int cv = tid + q * kPrefillThreads;
          const int64_t tile = int64_t(bl) * p.Hkv + col_h[q];
          float run[VEC];
#pragma unroll
          for (int e = 0; e < VEC; ++e) run[e] = 0.f;
#pragma unroll
          for (int k = 0; k < kMaxScales; ++k) {
            if (k >= a.kU) break;
#pragma unroll
            for (int e = 0; e < VEC; ++e) run[e] += acc[q][k][e];
            if (r1 == P) {  // the sequence's prefix ends here: open partial of scale k
              float* pp = p.part + ((tile * p.nsc + k) * 2 + col_t[q]) * p.D + col_d0[q];
#pragma unroll
              for (int e = 0; e < VEC; e += 4)
                *reinterpret_cast<float4*>(pp + e) = make_float4(run[e], run[e + 1], run[e + 2], run[e + 3]);
            }
          }
          if (!unit_closed) {
            float* w = a.ws + (int64_t(bl) * a.n_units + u) * (2 * rowElems) + int64_t(cv) * VEC;
#pragma unroll
            for (int e = 0; e < VEC; e += 4)
              *reinterpret_cast<float4*>(w + e) = make_float4(run[e], run[e + 1], run[e + 2], run[e + 3]);
          }
        }
      }
      ++consumed;
      cursor_next(a, p, cons);
    }
  }
}

// Pass 2: per (sequence*layer, column block of 64 column vectors).
template <typename T>
__global__ void __launch_bounds__(64)
prefill_finalize_kernel(Dev p, PrefillArgs a, const T* __restrict__ last_hidden) {
  using E = Elem<T>;
  constexpr int VEC = E::kVec;
  const int bl = blockIdx.x;
  const int b = bl / p.L;
  const int rowElems = p.Hkv * p.D;
  const int ncv = 2 * rowElems / VEC;
  const int cvPerRow = rowElems / VEC;
  const int cv = blockIdx.y * blockDim.x + threadIdx.x;
  int64_t* ctr = p.counters + int64_t(bl) * (1 + p.nsc);

  const int64_t Praw = a.prefix_len[b];
  const int64_t P = Praw < 0 ? 0 : Praw;
  const int64_t len_prev = ctr[0];
  const int64_t end = min(a.row_end, P);
  const int64_t smax = p.scales[p.nsc - 1];
  if (blockIdx.y == 0 && threadIdx.x == 0) {
    if (Praw < 0) set_err(p.err, LS_DEVERR_PREFIX_LEN);
    if (len_prev != min(a.row_begin, P)) set_err(p.err, LS_DEVERR_ORDER);
    if (P > a.row_end && a.row_end % smax != 0) set_err(p.err, LS_DEVERR_ORDER);
  }
  const int64_t newlen = end > a.row_begin ? end : len_prev;

  if (cv < ncv) {
    const int t = cv / cvPerRow;
    const int e0 = (cv - t * cvPerRow) * VEC;
    const int h = e0 / p.D, d0 = e0 - h * p.D;
    const int64_t tile = int64_t(bl) * p.Hkv + h;
    T* kvt = reinterpret_cast<T*>(p.kv) + (tile * 2 + t) * int64_t(p.R) * p.D;

    if (end > a.row_begin) {
      const int nu = int((end - a.row_begin + a.U - 1) / a.U);
      float acc[kMaxScales + 1][VEC], gs[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        gs[e] = 0.f;
#pragma unroll
        for (int k = 0; k <= kMaxScales; ++k) acc[k][e] = 0.f;
      }
      for (int uu = 0; uu < nu; ++uu) {
        const float* w = a.ws + (int64_t(bl) * a.n_units + uu) * (2 * rowElems) + int64_t(cv) * VEC;
        float x[VEC];
#pragma unroll
        for (int e = 0; e < VEC; e += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(w + e);
          x[e] = v4.x; x[e + 1] = v4.y; x[e + 2] = v4.z; x[e + 3] = v4.w;
        }
        if (a.kU >= p.nsc) {
#pragma unroll
          for (int e = 0; e < VEC; ++e) gs[e] += x[e];
          continue;
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[a.kU][e] += x[e];
        const int64_t eu = a.row_begin + int64_t(uu + 1) * a.U;  // row after this unit
        if (eu > end) continue;                                 // open unit
        for (int k = a.kU; k < p.nsc; ++k) {
          const int s = p.scales[k];
          if (eu % s != 0) break;
          const int64_t j = eu / s - 1;
          if (j >= P / s - p.slots) {
            float m[VEC];
#pragma unroll
            for (int e = 0; e < VEC; ++e) m[e] = acc[k][e] / float(s);
            const int slot = int(j % p.slots);
            float* sg = p.seg + (((tile * p.nsc + k) * p.slots + slot) * 2 + t) * p.D + d0;
#pragma unroll
            for (int e = 0; e < VEC; e += 4)
              *reinterpret_cast<float4*>(sg + e) = make_float4(m[e], m[e + 1], m[e + 2], m[e + 3]);
            *reinterpret_cast<uint4*>(kvt + (int64_t(p.W) + k * (p.slots + 1) + slot) * p.D + d0) =
                E::from_f32(m);
          }
          if (k + 1 < p.nsc) {
#pragma unroll
            for (int e = 0; e < VEC; ++e) { acc[k + 1][e] += acc[k][e]; acc[k][e] = 0.f; }
          } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) { gs[e] += acc[k][e]; acc[k][e] = 0.f; }
          }
        }
      }
      // open partials of the scales > U, then the rest of the global sum
      float run[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) run[e] = 0.f;
      for (int k = a.kU; k < p.nsc; ++k) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) run[e] += acc[k][e];
        if (end == P) {
          float* pp = p.part + ((tile * p.nsc + k) * 2 + t) * p.D + d0;
#pragma unroll
          for (int e = 0; e < VEC; e += 4)
            *reinterpret_cast<float4*>(pp + e) = make_float4(run[e], run[e + 1], run[e + 2], run[e + 3]);
        }
      }
      float* gp = p.glob + (tile * 2 + t) * p.D + d0;
#pragma unroll
      for (int e = 0; e < VEC; e += 4) {
        float4 v4 = *reinterpret_cast<const float4*>(gp + e);
        v4.x += gs[e] + run[e]; v4.y += gs[e + 1] + run[e + 1];
        v4.z += gs[e + 2] + run[e + 2]; v4.w += gs[e + 3] + run[e + 3];
        *reinterpret_cast<float4*>(gp + e) = v4;
      }
    }

    // mean rows of the partials and of the global sum for the attention
    float m[VEC];
    for (int k = 0; k < p.nsc; ++k) {
      const int64_t c = newlen % p.scales[k];
      const float* pp = p.part + ((tile * p.nsc + k) * 2 + t) * p.D + d0;
#pragma unroll
      for (int e = 0; e < VEC; ++e) m[e] = c > 0 ? pp[e] / float(c) : 0.f;
      *reinterpret_cast<uint4*>(kvt + (int64_t(p.W) + k * (p.slots + 1) + p.slots) * p.D + d0) =
          E::from_f32(m);
    }
    const float* gp = p.glob + (tile * 2 + t) * p.D + d0;
#pragma unroll
    for (int e = 0; e < VEC; ++e) m[e] = newlen > 0 ? gp[e] / float(newlen) : 0.f;
    *reinterpret_cast<uint4*>(kvt + int64_t(p.R - 1) * p.D + d0) = E::from_f32(m);
  }

  if (blockIdx.y == 0) {
    if (last_hidden != nullptr) {
      const T* src = last_hidden + int64_t(bl) * p.hidden;
      T* dst = reinterpret_cast<T*>(p.boundary) + int64_t(bl) * p.hidden;
      for (int x = threadIdx.x * VEC; x < p.hidden; x += blockDim.x * VEC)
        *reinterpret_cast<uint4*>(dst + x) = ld_nc_v4(src + x);
    }
    __syncthreads();  // every thread of this block has read ctr[0]
    if (threadIdx.x == 0) {
      ctr[0] = newlen;
      for (int k = 0; k < p.nsc; ++k) ctr[1 + k] = newlen / p.scales[k];
    }
  }
}

// ---- host side -------------------------------------------------------------------
struct PrefillPlan {
  int32_t U, kU, G, n_units;
};

PrefillPlan prefill_plan(const ls_config& c, int64_t row_begin, int64_t row_end) {
  PrefillPlan pl{};
  int kU = 0;
  for (int k = 0; k < c.n_scales; ++k)
    if (c.scales[k] <= 512) kU = k + 1;
  if (kU == 0) kU = 1;
  pl.kU = kU;
  pl.U = c.scales[kU - 1];
  const int elem = c.dtype == LS_BF16 ? 2 : 4;
  const int rowBytes = c.n_kv_heads * c.head_dim * elem;
  pl.G = max(1, min(64, 32768 / rowBytes));
  const int64_t rows = row_end > row_begin ? row_end - row_begin : 0;
  pl.n_units = int32_t((rows + pl.U - 1) / pl.U);
  return pl;
}

size_t prefill_workspace_bytes(const ls_config& c, int64_t row_begin, int64_t row_end) {
  const PrefillPlan pl = prefill_plan(c, row_begin, row_end);
  return size_t(c.batch) * c.n_layers * size_t(pl.n_units) * 2 * c.n_kv_heads * c.head_dim * 4 + 256;
}

template <typename T, int CVT, typename Src>
static cudaError_t launch_units(const Dev& p, const PrefillArgs& a, const Src& src, int sms, cudaStream_t stream) {
  const int rowBytes = p.Hkv * p.D * int(sizeof(T));
  const size_t smem = size_t(kPrefillStages) * 2 * a.G * rowBytes;
  auto kern = prefill_units_kernel<T, CVT, Src>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int grid = max(1, min(a.n_items, sms));
  kern<<<grid, kPrefillBlock, smem, stream>>>(p, a, src);
  return cudaGetLastError();
}

template <typename Src>
static cudaError_t launch_prefill_src(const Dev& p, const ls_config& c, const void* k, const void* v,
                                      int64_t plane_stride, int64_t row_stride, const Src& src,
                                      const int64_t* prefix_len, int64_t row_begin, int64_t row_end,
                                      const void* last_hidden, void* ws, int sms, cudaStream_t stream) {
  const PrefillPlan pl = prefill_plan(c, row_begin, row_end);
  PrefillArgs a{};
  a.k = static_cast<const char*>(k);
  a.v = static_cast<const char*>(v);
  a.plane_stride = plane_stride;
  a.row_stride = row_stride;
  a.prefix_len = prefix_len;
  a.row_begin = row_begin;
  a.row_end = row_end;
  a.ws = static_cast<float*>(ws);
  a.n_units = pl.n_units;
  a.U = pl.U;
  a.kU = pl.kU;
  a.G = pl.G;
  a.n_items = p.b * p.L * pl.n_units;
  const int vec = p.dtype == LS_BF16 ? 8 : 4;
  const int ncv = 2 * p.Hkv * p.D / vec;
  const int cvt = (ncv + kPrefillThreads - 1) / kPrefillThreads;
  cudaError_t e = cudaSuccess;
  if (a.n_items > 0) {
    if (p.dtype == LS_BF16) {
      if (cvt <= 1) e = launch_units<__nv_bfloat16, 1>(p, a, src, sms, stream);
      else if (cvt <= 2) e = launch_units<__nv_bfloat16, 2>(p, a, src, sms, stream);
      else e = launch_units<__nv_bfloat16, 4>(p, a, src, sms, stream);
    } else {
      if (cvt <= 1) e = launch_units<float, 1>(p, a, src, sms, stream);
      else if (cvt <= 2) e = launch_units<float, 2>(p, a, src, sms, stream);
      else e = launch_units<float, 4>(p, a, src, sms, stream);
    }
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(p.b * p.L, (ncv + 63) / 64);
  if (p.dtype == LS_BF16)
    prefill_finalize_kernel<__nv_bfloat16><<<grid, 64, 0, stream>>>(
        p, a, static_cast<const __nv_bfloat16*>(last_hidden));
  else
    prefill_finalize_kernel<float><<<grid, 64, 0, stream>>>(p, a, static_cast<const float*>(last_hidden));
  return cudaGetLastError();
}

cudaError_t launch_prefill(const Dev& p, const ls_config& c, const void* k, const void* v,
                           int64_t plane_stride, int64_t row_stride, const int64_t* prefix_len,
                           int64_t row_begin, int64_t row_end, const void* last_hidden, void* ws,
                           int sms, cudaStream_t stream) {
  return launch_prefill_src(p, c, k, v, plane_stride, row_stride, DensePrefix{}, prefix_len, row_begin, row_end,
                            last_hidden, ws, sms, stream);
}

cudaError_t launch_prefill_paged(const Dev& p, const ls_config& c, const ls_paged_kv& kv, const int64_t* prefix_len,
                                 int64_t row_begin, int64_t row_end, const void* last_hidden, void* ws, int sms,
                                 cudaStream_t stream) {
  return launch_prefill_src(p, c, nullptr, nullptr, 0, 0, kv, prefix_len, row_begin, row_end, last_hidden, ws,
                            sms, stream);
}

// ---- fixed scratch for callers that cannot allocate ----------------------------------
// The unit sums of pass 1 live here instead of in a caller workspace. Every GPU that
// loads the library holds this array until the process exits. Nothing in it has to start
// at zero: pass 2 only reads unit sums that pass 1 of the same call wrote. Calls share it,
// so calls that overlap on the GPU race.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of the array on `device`, which must be the current device (the entry
// points check that the state's device is current), looked up once per device: the
// host-side name of the array is not a device address.
cudaError_t noalloc_scratch(int device, void** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return e;
  if (device != cur || device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[device]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[device] = p;
  }
  *out = addr[device];
  return cudaSuccess;
}

}  // namespace ls
