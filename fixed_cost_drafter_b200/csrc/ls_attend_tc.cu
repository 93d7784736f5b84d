// Drafter block attention over the three views on the 5th-generation tensor cores:
// LongSpark paper page, Figure 2 caption (c): the drafter attends over fixed-size views,
// so its cost does not depend on the prefix length.
//
// One tile = (sequence, layer, KV head g): M = (Hq/Hkv) * B = 64 query rows (the GQA
// group's heads x the block's queries, row m = i * group + j) against the tile's
// kv_rows arena rows (ring window + summary mean rows) followed by the boundary row:
// R + 1 <= 768 key/value rows stream through in chunks of 128 with an online softmax. The
// boundary row (a per-tile vector given by the caller) is written by the producer warps
// into the last chunk's stage right after the tile's rows, so every row of the views is
// handled the same way.
//
// Persistent kernel, one CTA per SM, 12 warps; the roles only meet at mbarriers, so no
// role's order of work can hold up another's:
//   warp 0    TMA producer of Q (3-D tensor map, two 64-column swizzled halves) and of
//             the K rows of every chunk (ring of 3 K stages, tensor map over the arena),
//             plus the boundary key row.
//   warp 6    TMA producer of the V rows of every chunk (its own ring of 3 stages), plus
//             the boundary value row.
//   warp 1    TMEM allocator and the QK-issuing thread (tcgen05.mma kind::f16, bf16 in,
//             fp32 accumulate, M = 64). The M = 64 accumulator fills lanes 0-15 of each
//             32-lane TMEM subpartition; a second accumulator at lane offset 16 fills
//             lanes 16-31. S_c = Q K_c^T is issued as two N = 64 halves (keys 0-63 to
//             lanes 0-15, keys 64-127 to lanes 16-31 of the same 64 columns), so the two
//             threads of a row pair each own half of the chunk's keys. Four S buffers.
//   warp 7    the PV-issuing thread: P_c V_c accumulates into the tile's output O, split
//             over the output columns the same way; O is double-buffered by tile. P is the
//             MMA's A operand straight from TMEM (two P buffers), V its B operand in shared
//             memory. 512 TMEM columns in all: S 0-255, O 256-383, P 384-511.
//   warps 2-5 softmax, one TMEM subpartition each, thread pairs (t, t+16) per query row.
//             Per chunk: the chunk's key mask (from a table the epilogue warps fill one
//             tile ahead), scaled logits, row max, exp2 against the row's reference max,
//             bf16 P into TMEM (a row's 128 keys as 64 packed columns of its lane, once in
//             lanes 0-15 and once in lanes 16-31 for the two output halves). The
//             reference max only moves when a chunk exceeds it by more than 2^8 (then the
//             row's O in TMEM and its running sum are rescaled once), so no chunk's P V
//             has to come back to registers. After a tile's last chunk the row sums go
//             to the epilogue warps through shared memory.
//   warps 8-11 epilogue, one TMEM subpartition each: O of a tile from TMEM (O is
//             double-buffered by tile) times 1/rowsum, to global memory, while the
//             softmax warps already work on the next tile. A bf16 O goes through the
//             tile's own Q buffer (free once its last P V has landed) and leaves with one
//             TMA tensor store, so no global store instruction competes with the softmax's
//             exp2 for the SM sub-partitions' shared-function queue. Warp 8 also turns the
//             counters of the tile two ahead into the key masks of its chunks.
// Every launch is programmatically dependent on the kernel before it on the stream: the
// kernel allocates TMEM and sets up its barriers, then every thread waits on the device
// (griddepcontrol.wait) before it reads what that kernel may have written, and triggers
// its own dependents right after the wait (so a kernel launched behind this one starts
// only once the kernel before this one has completed). ls_round launches it behind the
// commit kernel, whose trigger comes once its loads are in flight: the first tile's Q
// (complete before the commit started) is loaded before the wait. When no call has
// written the views since an attention launched on the same stream (a drafter's
// per-layer calls), the producers issue the first tile's first K/V chunks before the
// wait, so one launch's pipeline fills while the launch before it drains.
// Every wait is bounded and warp-uniform; a wait that runs out sets
// LS_DEVERR_WAIT_TIMEOUT, all roles stop, the copies in flight land, TMEM is freed.
#include <cuda.h>

#include "ls_attend_tc.h"
#include "ls_tc.cuh"

namespace ls {

namespace {

constexpr int kKStages = 3;           // K ring
constexpr int kVStages = 3;           // V ring
constexpr int kChunk = 128;            // arena rows per chunk
constexpr int kMaxChunks = 6;          // kv_rows + 1 <= 768
constexpr int kThreads = 384;          // 12 warps: 3 per SM sub-partition, <= 168 registers
constexpr int kQBytes = 64 * 128 * 2;  // one Q tile (two 8 KB halves)
constexpr int kStageBytes = kChunk * 128 * 2;  // one K or V chunk (two 16 KB halves: d 0-63 / 64-127)
constexpr int kSmemBytes = 2 * kQBytes + (kKStages + kVStages) * kStageBytes + 1024;
constexpr int kSBufs = 4;              // S buffers: QK may run up to four chunks ahead
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 256;        // O buffers at columns 256 + 64 * (tile & 1)
constexpr uint32_t kPCol = 384;        // P buffers at columns 384 + 64 * (chunk & 1)
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P values stay <= 2^8

struct TcArgs {
  int32_t lb, lcount, n_tiles;
  int32_t n_chunks;   // chunks per tile: floor(R / 128) + 1, the last holding the boundary row
  int32_t tail_rows;  // R mod 128: the tile's arena rows in its last chunk
  const __nv_bfloat16* bk;
  const __nv_bfloat16* bv;
  int64_t bstride;
  float scale_log2;  // softmax_scale * log2(e)
  void* out;         // bf16, or fp32 when Dev::out_f32
  int32_t views;         // LS_VIEW_* taking part in the softmax
  uint32_t chunk_mask;   // bit c: chunk c is streamed (the last chunk always is)
  int32_t tail_load;     // the last chunk's arena rows are loaded (else only its boundary row)
  int32_t mode;          // AttendLaunch: what may be read before the grid dependency wait
};

// Chunks streamed after chunk c (c = -1: the first one): nC or more when none is left.
__device__ inline int next_chunk(uint32_t mask, int c) {
  const uint32_t m = mask >> (c + 1);
  return m ? c + __ffs(int(m)) : 32;
}

struct Bars {
  uint64_t kfull[kKStages], kempty[kKStages];
  uint64_t vfull[kVStages], vempty[kVStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[kSBufs], s_free[kSBufs];
  uint64_t p_full[2], p_empty[2];
  uint64_t pv_done;
  uint64_t o_full[2], o_free[2];
  uint64_t lsum_full[2], lsum_free[2];
  uint64_t info_full[2], info_free[2];
  uint64_t o_staged;
  float lsum_buf[2][64];  // row sums of the last two tiles, softmax -> epilogue
  uint64_t vmask[2][kMaxChunks][2];  // key masks of the last two tiles: [chunk][64-row half]
  uint32_t tmem_base;
  uint32_t abort;
};

// 16 lanes from taddr on: lanes 0-15 of the warp write columns 0-31 of their lane, lanes
// 16-31 columns 32-63 of the same 16 lanes (the 16x32bx2 shape, half split at 32 columns).
__device__ inline void tmem_st_pairs(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], 32, {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ inline float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


// Bounded wait that also gives up when another role has already aborted.
__device__ inline bool wait_or_abort(Bars& s, uint64_t* bar, uint32_t parity, int32_t* err) {
#pragma unroll 1  // one copy per call site: the kernel's code must stay small for the instruction cache
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023) == 1023 && *reinterpret_cast<volatile uint32_t*>(&s.abort)) return false;
  }
  set_err(err, LS_DEVERR_WAIT_TIMEOUT);
  *reinterpret_cast<volatile uint32_t*>(&s.abort) = 1;
  return false;
}

__device__ inline void tile_coords(int t, const Dev& p, int lcount, int& b, int& lc, int& g) {
  g = t % p.Hkv;
  const int rest = t / p.Hkv;
  lc = rest % lcount;
  b = rest / lcount;
}

// Validity of the 64 rows [r0, r0 + 64) of a tile's key/value stream as a bit mask
// (bit i = row r0 + i). The stream is the tile's arena rows followed by the boundary row
// (row R): ring slots below min(len, W), per scale the first min(n_seg, slots) segment
// slots and the partial mean when its segment is non-empty, the global mean when len > 0,
// and the boundary row always; then only the rows of the views in `views` (LS_VIEW_*).
__device__ inline uint64_t range_bits(int lo, int hi, int r0) {
  lo = max(lo, r0);
  hi = min(hi, r0 + 64);
  if (hi <= lo) return 0ull;
  const int n = hi - lo;
  const uint64_t m = n >= 64 ? ~0ull : ((1ull << n) - 1ull);
  return m << (lo - r0);
}
// sinfo: 16 bits per scale k at bit 16k: valid segment slots (bits 0-14), partial non-empty (bit 15).
__device__ inline uint64_t view_mask(const Dev& p, int r0, int ring_valid, uint64_t sinfo, bool has_glob,
                                    int views) {
  uint64_t m = (views & LS_VIEW_WINDOW) ? range_bits(0, ring_valid, r0) : 0ull;
  int base = p.W;
  if (views & LS_VIEW_SUMMARY) {
#pragma unroll 1
    for (int k = 0; k < p.nsc; ++k) {
      const uint32_t e = uint32_t(sinfo >> (16 * k));
      m |= range_bits(base, base + int(e & 0x7fffu), r0);
      if (e & 0x8000u) m |= range_bits(base + p.slots, base + p.slots + 1, r0);
      base += p.slots + 1;
    }
    if (has_glob) m |= range_bits(base, base + 1, r0);  // global mean, row R - 1
  }
  if (views & LS_VIEW_BOUNDARY) m |= range_bits(p.R, p.R + 1, r0);  // boundary row, row R
  return m;
}

// Work of one CTA: tiles blockIdx.x, blockIdx.x + gridDim.x, ... (each all nC chunks).
__device__ inline int item_count(const TcArgs& a) {
  return blockIdx.x < a.n_tiles ? (a.n_tiles - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
}
__device__ inline int item_tile(int i) { return int(blockIdx.x) + i * int(gridDim.x); }

// kOutF32: fp32 output written with plain stores; otherwise bf16 output through a TMA store.
template <bool kOutF32>
__global__ void __launch_bounds__(kThreads, 1)
attend_tc_kernel(const Dev p, const TcArgs a, const __grid_constant__ CUtensorMap kv_map,
                 const __grid_constant__ CUtensorMap kv_tail_map, const __grid_constant__ CUtensorMap q_map,
                 const __grid_constant__ CUtensorMap o_map) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ Bars s;
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_buf = smem;                           // [2][kQBytes]
  unsigned char* k_buf = q_buf + 2 * kQBytes;            // [kKStages][kStageBytes]
  unsigned char* v_buf = k_buf + kKStages * kStageBytes; // [kVStages][kStageBytes]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nC = a.n_chunks;
  const int tail = a.tail_rows;                   // the tile's arena rows in its last chunk
  const int last_rows = (tail + 1 + 15) & ~15;    // rows the last chunk's MMAs take (+ boundary)
  const int n_items = item_count(a);
  const int c_first = next_chunk(a.chunk_mask, -1);  // chunks of left-out views are skipped

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKStages; ++i) { mbar_init(&s.kfull[i], 1); mbar_init(&s.kempty[i], 1); }
    for (int i = 0; i < kVStages; ++i) { mbar_init(&s.vfull[i], 1); mbar_init(&s.vempty[i], 1); }
    for (int i = 0; i < kSBufs; ++i) { mbar_init(&s.s_full[i], 1); mbar_init(&s.s_free[i], 128); }
    for (int i = 0; i < 2; ++i) {
      // a Q buffer is free once its tile's QK is done and, for a bf16 output, once the
      // tile's O staged in it has been read by the TMA store
      mbar_init(&s.q_full[i], 1); mbar_init(&s.q_empty[i], kOutF32 ? 1 : 2);
      mbar_init(&s.info_full[i], 32); mbar_init(&s.info_free[i], 128);
      mbar_init(&s.p_full[i], 128); mbar_init(&s.p_empty[i], 1);
      mbar_init(&s.o_full[i], 1); mbar_init(&s.o_free[i], 128);
      mbar_init(&s.lsum_full[i], 128); mbar_init(&s.lsum_free[i], 128);
    }
    mbar_init(&s.pv_done, 1);
    mbar_init(&s.o_staged, 128);
    s.abort = 0;
    fence_mbar_init();
  }
  {
    // rows of the last chunk past the boundary row are read by its MMAs (masked): they
    // must hold finite values, zeros until a full chunk has used the stage
    // (with the last chunk's arena rows not loaded, all of its rows but the boundary row)
    const int z0 = a.tail_load ? tail + 1 : 0;
    const int zr = last_rows - z0;
    if (zr > 0) {
      const int n = (kKStages + kVStages) * 2 * zr * 8;
      for (int i = threadIdx.x; i < n; i += kThreads) {
        const int piece = i & 7, r = z0 + (i >> 3) % zr, sh = (i >> 3) / zr;
        *reinterpret_cast<uint4*>(k_buf + sh * (kStageBytes / 2) + r * 128 + piece * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  // Every thread passes the grid dependency wait before it triggers this grid's dependents;
  // the producers (warps 0, 6) and the mask warp (8) do both in their roles, after what
  // they may read before the wait. The other roles need data only those roles bring.
  const bool no_wait = a.mode == kAttendFree;  // nothing this kernel reads is the kernel before's
  if (warp != 0 && warp != 6 && warp != 8) {
    if (!no_wait) grid_dependency_wait();
    allow_dependent_launch();
  }
  int issued = 0;  // producers: loads issued into their ring (for the drain after an abort)
  auto chunk_rows = [&](int c) { return c == nC - 1 ? last_rows : kChunk; };

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------ producers
    // The whole warp runs the loop; lane 0 issues the copies. Lanes 0-15 carry the tile's
    // boundary row (16 bytes each), loaded when the tile starts and written into the
    // last chunk's stage right after the tile's rows, in the TMA's 128-byte swizzle.
    const bool is_k = warp == 0;
    const int nst = is_k ? kKStages : kVStages;
    uint64_t* fullb = is_k ? s.kfull : s.vfull;
    uint64_t* emptyb = is_k ? s.kempty : s.vempty;
    unsigned char* ring = is_k ? k_buf : v_buf;
    const __nv_bfloat16* bsrc = is_k ? a.bk : a.bv;
    if (lane == 0) {
      prefetch_map(&kv_map);
      if (tail > 0) prefetch_map(&kv_tail_map);
      if (is_k) prefetch_map(&q_map);
    }
    const int grp = p.Hq / p.Hkv;
    // Q of item i into its buffer (the K producer's job)
    auto load_q = [&](int i, int b, int lc, int g) -> bool {
      const int qb = i & 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(s, &s.q_empty[qb], ((i >> 1) & 1) ^ 1, p.err))) return false;
      if (lane == 0) {
        mbar_arrive_expect_tx(&s.q_full[qb], kQBytes);
        const int zrow = (b * a.lcount + lc) * p.B;
        tma_load_3d(q_buf + qb * kQBytes, &q_map, 0, g * grp, zrow, &s.q_full[qb]);
        tma_load_3d(q_buf + qb * kQBytes + kQBytes / 2, &q_map, 64, g * grp, zrow, &s.q_full[qb]);
      }
      return true;
    };
    // one chunk's arena rows into stage st (lane 0 issues)
    auto load_chunk = [&](int64_t tile, int c, int st) {
      if (lane == 0) {
        const bool last = c == nC - 1;
        const int rows = last ? (a.tail_load ? tail : 0) : kChunk;
        mbar_arrive_expect_tx(&fullb[st], uint32_t(rows * 256));
        if (rows > 0) {
          const CUtensorMap* m = last ? &kv_tail_map : &kv_map;
          const int y = int((tile * 2 + (is_k ? 0 : 1)) * p.R + int64_t(c) * kChunk);
          unsigned char* dst = ring + st * kStageBytes;
          tma_load_2d(dst, m, 0, y, &fullb[st]);
          tma_load_2d(dst + kStageBytes / 2, m, 64, y, &fullb[st]);
        }
      }
    };
    bool ok = true;
    int pre = 0;  // chunks of the first tile issued before the grid dependency wait
    if (a.mode == kAttendViewsSettled && n_items > 0) {
      // the views are complete: the first tile's chunks that fit the empty ring (the last
      // chunk waits: it carries the caller's boundary row)
      int b, lc, g;
      tile_coords(item_tile(0), p, a.lcount, b, lc, g);
      const int64_t tile = (int64_t(b) * p.L + (a.lb + lc)) * p.Hkv + g;
      for (int c = c_first; c < nC - 1 && pre < nst; c = next_chunk(a.chunk_mask, c)) {
        load_chunk(tile, c, pre);  // stage `pre`: the ring is empty at the start
        ++pre;
        ++issued;
      }
    }
    if (is_k && a.mode == kAttendAfterCommit && n_items > 0) {
      // Q is an input complete before the commit started; the boundary rows and the
      // arena are state the commit writes
      int b, lc, g;
      tile_coords(item_tile(0), p, a.lcount, b, lc, g);
      ok = load_q(0, b, lc, g);
    }
    if (!no_wait) grid_dependency_wait();
    allow_dependent_launch();
    int k = 0;  // chunks of this CTA so far: ring stage and phase
    for (int i = 0; i < n_items && ok; ++i) {
      int b, lc, g;
      tile_coords(item_tile(i), p, a.lcount, b, lc, g);
      const int64_t tile = (int64_t(b) * p.L + (a.lb + lc)) * p.Hkv + g;
      if (is_k && !(i == 0 && a.mode == kAttendAfterCommit)) {  // Q of the item first
        if (!load_q(i, b, lc, g)) break;
      }
      // the boundary row is loaded once the tile's first chunk is on its way (its latency
      // then overlaps the stream), or before a one-chunk tile's only chunk
      const __nv_bfloat16* bptr = bsrc + (int64_t(b) * p.L + (a.lb + lc)) * a.bstride + g * 128 + lane * 8;
      uint4 brow = make_uint4(0, 0, 0, 0);
      for (int c = c_first; c < nC; c = next_chunk(a.chunk_mask, c), ++k) {
        const int st = k % nst;
        const bool last = c == nC - 1;
        if (k < pre) {  // issued before the wait
          if (c == c_first && !last && lane < 16) brow = ld_nc_v4(bptr);
          continue;
        }
        if (!__all_sync(0xffffffffu, wait_or_abort(s, &emptyb[st], ((k / nst) & 1) ^ 1, p.err))) { ok = false; break; }
        unsigned char* dst = ring + st * kStageBytes;
        if (last) {  // the boundary row, row `tail` of the stage
          if (c == c_first && lane < 16) brow = ld_nc_v4(bptr);
          if (lane < 16)
            *reinterpret_cast<uint4*>(dst + (lane >> 3) * (kStageBytes / 2) + tail * 128 +
                                      (((lane & 7) ^ (tail & 7)) << 4)) = brow;
          fence_proxy_async_smem();
          __syncwarp();
        }
        load_chunk(tile, c, st);
        if (c == c_first && !last && lane < 16) brow = ld_nc_v4(bptr);
        ++issued;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ QK issuer
    if (lane == 0) {
      // descriptors of the buffers' first bytes; an operand further in adds its offset / 16
      // to the start-address field (shared addresses stay below 256 KB: no carry out)
      const uint64_t dq0 = sdesc(smem_u32(q_buf), 16, 1024), dk0 = sdesc(smem_u32(k_buf), 16, 1024);
      bool ok = true;
      int k = 0;
      for (int i = 0; i < n_items && ok; ++i) {
        const int qb = i & 1;
        if (!wait_or_abort(s, &s.q_full[qb], (i >> 1) & 1, p.err)) break;
        for (int c = c_first; c < nC; c = next_chunk(a.chunk_mask, c), ++k) {
          const int sb = k % kSBufs, st = k % kKStages;
          if (!wait_or_abort(s, &s.kfull[st], (k / kKStages) & 1, p.err)) { ok = false; break; }
          if (!wait_or_abort(s, &s.s_free[sb], ((k / kSBufs) & 1) ^ 1, p.err)) { ok = false; break; }
          tc_fence_after();
          const int rows = chunk_rows(c);
          const int n0 = rows < 64 ? rows : 64, n1 = rows - n0;
          const uint32_t id0 = idesc_bf16(n0, false), id1 = idesc_bf16(n1 > 0 ? n1 : 16, false);
          const uint64_t dq = dq0 + uint32_t(qb * kQBytes >> 4), dk = dk0 + uint32_t(st * kStageBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t qo = ((kk >> 2) * (kQBytes / 2) + (kk & 3) * 32) >> 4;
            const uint32_t ko = ((kk >> 2) * (kStageBytes / 2) + (kk & 3) * 32) >> 4;
            mma_bf16(tmem + 64 * sb, dq + qo, dk + ko, id0, kk > 0);
            if (n1 > 0) mma_bf16(tmem + (16u << 16) + 64 * sb, dq + qo, dk + ko + (64 * 128 >> 4), id1, kk > 0);
          }
          mma_commit(&s.kempty[st]);
          mma_commit(&s.s_full[sb]);
          if (c == nC - 1) mma_commit(&s.q_empty[qb]);
        }
      }
    }
  } else if (warp == 7) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0) {
      const uint64_t dv0 = sdesc(smem_u32(v_buf), kStageBytes / 2, 1024);
      const uint32_t id_pv = idesc_bf16(64, true);
      bool ok = true;
      int k = 0;
      for (int i = 0; i < n_items && ok; ++i) {
        const int ob = i & 1;
        if (!wait_or_abort(s, &s.o_free[ob], ((i >> 1) & 1) ^ 1, p.err)) break;
        for (int c = c_first; c < nC; c = next_chunk(a.chunk_mask, c), ++k) {
          const int pb = k & 1, st = k % kVStages;
          if (!wait_or_abort(s, &s.vfull[st], (k / kVStages) & 1, p.err)) { ok = false; break; }
          if (!wait_or_abort(s, &s.p_full[pb], (k >> 1) & 1, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dv = dv0 + uint32_t(st * kStageBytes >> 4);
          const uint32_t pa = tmem + kPCol + 64 * pb;  // 16 keys = 8 packed columns per step
          const int rows = chunk_rows(c);
          for (int kk = 0; kk < rows / 16; ++kk) {
            const uint32_t acc = (c != c_first || kk > 0) ? 1u : 0u;
            // V: rows = keys (K dim), 128-byte rows per 64-column half: MN-major B, SBO = 8 rows
            mma_bf16_ta(tmem + kOCol + 64 * ob, pa + 8 * kk, dv + uint32_t(kk * 2048 >> 4), id_pv, acc);
            mma_bf16_ta(tmem + (16u << 16) + kOCol + 64 * ob, pa + (16u << 16) + 8 * kk,
                        dv + uint32_t((kStageBytes / 2 + kk * 2048) >> 4), id_pv, acc);
          }
          mma_commit(&s.vempty[st]);
          mma_commit(&s.p_empty[pb]);
          mma_commit(&s.pv_done);
          if (c == nC - 1) mma_commit(&s.o_full[ob]);
        }
      }
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ softmax
    const int sub = warp & 3;           // TMEM subpartition this warp may access
    const int half = lane >> 4;         // 0: keys / output columns 0-63, 1: 64-127
    const int row = 16 * sub + (lane & 15);
    const uint32_t trow = tmem + (uint32_t(32 * sub) << 16);
    const float sl2 = a.scale_log2;     // > 0 (checked by the caller)
    int k = 0;
    for (int i = 0; i < n_items; ++i) {
      const int ob = i & 1;
      // the key masks of this tile's chunks (epilogue warp 8 fills them from the counters)
      if (!__all_sync(0xffffffffu, wait_or_abort(s, &s.info_full[ob], (i >> 1) & 1, p.err))) break;
      float mref = -INFINITY;  // reference max (log2 units) the P values are taken against
      float lsum = 0.f;        // sum of the rows' weights against mref
      bool ok = true;
      for (int c = c_first; c < nC; c = next_chunk(a.chunk_mask, c), ++k) {
        const int sb = k % kSBufs, pb = k & 1;
        const uint64_t vm = s.vmask[ob][c][half];
        const bool all_valid = __all_sync(0xffffffffu, vm == ~0ull);
        if (!__all_sync(0xffffffffu, wait_or_abort(s, &s.s_full[sb], (k / kSBufs) & 1, p.err))) { ok = false; break; }
        tc_fence_after();
        float sv[64];
        tmem_ld32(trow + 64 * sb, sv);
        tmem_ld32(trow + 64 * sb + 32, sv + 32);
        tc_fence_before();
        mbar_arrive(&s.s_free[sb]);
        // row max over the valid raw logits (scale > 0 keeps the order), 8-way tree
        float mx8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
        if (all_valid) {
#pragma unroll
          for (int e = 0; e < 64; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], sv[e]);
        } else {
#pragma unroll
          for (int e = 0; e < 64; ++e) {
            if (!((vm >> e) & 1ull)) sv[e] = -INFINITY;
            mx8[e & 7] = fmaxf(mx8[e & 7], sv[e]);
          }
        }
        float cmax = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                           fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 16)) * sl2;
        // P buffer pb free again means P_{k-2} V_{k-2} has landed; only after that does the
        // parity wait on pv_done below identify P_{k-1} V_{k-1} unambiguously
        if (!__all_sync(0xffffffffu, wait_or_abort(s, &s.p_empty[pb], ((k >> 1) & 1) ^ 1, p.err))) { ok = false; break; }
        if (c == c_first) {
          mref = cmax;  // O is still empty: the reference moves for free
        } else if (__any_sync(0xffffffffu, cmax > mref + kRescaleThreshold)) {
          // rows whose max grew by more than 2^8: rescale their O (after the P V MMAs
          // issued so far have landed) and their running sum to the new reference
          const float mnew = cmax > mref + kRescaleThreshold ? cmax : mref;
          const float alpha = ex2(mref - mnew);  // 0 while no row was valid yet
          if (!__all_sync(0xffffffffu, wait_or_abort(s, &s.pv_done, (k - 1) & 1, p.err))) { ok = false; break; }
          tc_fence_after();
          float ov[32];
#pragma unroll 1
          for (int h2 = 0; h2 < 2; ++h2) {
            tmem_ld32(trow + kOCol + 64 * ob + 32 * h2, ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] *= alpha;
            tmem_st32(trow + kOCol + 64 * ob + 32 * h2, ov);
          }
          tc_fence_before();
          lsum *= alpha;
          mref = mnew;
        }
        // weights 2^(s * scale - mref) (masked slots hold -inf: weight 0), bf16 P, 8-way sums;
        // before any valid row the reference is -inf and every slot so far is masked
        const float mu = mref == -INFINITY ? 0.f : mref;
        float ps8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) ps8[u] = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float p0 = ex2(fmaf(sv[e], sl2, -mu));
          const float p1 = ex2(fmaf(sv[e + 1], sl2, -mu));
          ps8[(e >> 1) & 7] += p0 + p1;
          pk[e >> 1] = pack_bf16(p0, p1);
        }
        const float psum = ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
        lsum += psum + __shfl_xor_sync(0xffffffffu, psum, 16);
        // the row's 128 keys as 64 packed columns (this thread's 64 keys at columns
        // 32 * half ...), in lanes 0-15 and again in lanes 16-31 of the subpartition
        tmem_st_pairs(trow + kPCol + 64 * pb, pk);
        tmem_st_pairs(trow + (16u << 16) + kPCol + 64 * pb, pk);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        mbar_arrive(&s.p_full[pb]);
      }
      if (!ok) break;
      mbar_arrive(&s.info_free[ob]);
      // the row sum goes to the epilogue warps, which read this tile's O once its last
      // P V has landed; the softmax goes on with the next tile
      if (!__all_sync(0xffffffffu, wait_or_abort(s, &s.lsum_free[ob], ((i >> 1) & 1) ^ 1, p.err))) break;
      if (half == 0) s.lsum_buf[ob][row] = lsum;
      mbar_arrive(&s.lsum_full[ob]);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ epilogue
    // Each thread owns an output slice (row, half): 64 columns of one row.
    const int sub = warp & 3;
    const int half = lane >> 4;
    const int row = 16 * sub + (lane & 15);
    const uint32_t trow = tmem + (uint32_t(32 * sub) << 16);
    const int grp = p.Hq / p.Hkv;
    // Warp 8: key masks of item i's chunks into table slot i & 1. Lane 2c + h takes the
    // 64 rows [128 c + 64 h, +64) of the tile's key/value stream (see view_mask).
    auto fill_masks = [&](int i) {
      int b, lc, g;
      tile_coords(item_tile(i), p, a.lcount, b, lc, g);
      const int64_t* ctr = p.counters + (int64_t(b) * p.L + a.lb + lc) * (1 + p.nsc);
      const int64_t len = ctr[0];
      uint64_t sinfo = 0;
#pragma unroll 1
      for (int kk = 0; kk < p.nsc; ++kk) {
        const int64_t n = ctr[1 + kk];
        const uint64_t e = uint64_t(n < p.slots ? n : int64_t(p.slots)) |
                           (len - n * p.scales[kk] > 0 ? 0x8000ull : 0ull);
        sinfo |= e << (16 * kk);
      }
      if (lane < 2 * nC)
        s.vmask[i & 1][lane >> 1][lane & 1] =
            view_mask(p, 64 * lane, len < p.W ? int(len) : p.W, sinfo, len > 0, a.views);
    };
    if (warp == 8) {
      // the counters are state a commit before this kernel writes, unless the views are
      // settled
      const bool early = a.mode == kAttendViewsSettled || no_wait;
      if (!early) {
        grid_dependency_wait();
        allow_dependent_launch();
      }
      for (int i = 0; i < 2 && i < n_items; ++i) {
        fill_masks(i);
        mbar_arrive(&s.info_full[i]);
      }
      if (early) {
        if (!no_wait) grid_dependency_wait();
        allow_dependent_launch();
      }
    }
    for (int i = 0; i < n_items; ++i) {
      int b, lc, g;
      tile_coords(item_tile(i), p, a.lcount, b, lc, g);
      const int ob = i & 1;
      if (!__all_sync(0xffffffffu, wait_or_abort(s, &s.lsum_full[ob], (i >> 1) & 1, p.err))) break;
      const float lsum = s.lsum_buf[ob][row];  // the boundary row is one of the summed rows
      mbar_arrive(&s.lsum_free[ob]);
      if (!__all_sync(0xffffffffu, wait_or_abort(s, &s.o_full[ob], (i >> 1) & 1, p.err))) break;
      tc_fence_after();
      float o[64];
      tmem_ld32(trow + kOCol + 64 * ob, o);
      tmem_ld32(trow + kOCol + 64 * ob + 32, o + 32);
      tc_fence_before();
      mbar_arrive(&s.o_free[ob]);
      const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;  // no valid row in the views: zeros
      const int zrow = (b * a.lcount + lc) * p.B;  // the tile's first query of the block
      if constexpr (kOutF32) {
        const int qi = row / grp, jj = row - qi * grp;
        float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(a.out) +
                                               ((int64_t(zrow) + qi) * p.Hq + g * grp + jj) * 128 + 64 * half);
#pragma unroll
        for (int u = 0; u < 16; ++u)
          o4[u] = make_float4(o[4 * u] * inv, o[4 * u + 1] * inv, o[4 * u + 2] * inv, o[4 * u + 3] * inv);
      } else {
        // O into the tile's Q buffer (row m = i_q * group + j, two swizzled 64-column
        // halves: the layout of the output tensor map's box), then one TMA store
        unsigned char* orow = q_buf + ob * kQBytes + half * (kQBytes / 2) + row * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<uint4*>(orow + ((u ^ (row & 7)) << 4)) =
              make_uint4(pack_bf16(o[8 * u] * inv, o[8 * u + 1] * inv), pack_bf16(o[8 * u + 2] * inv, o[8 * u + 3] * inv),
                         pack_bf16(o[8 * u + 4] * inv, o[8 * u + 5] * inv),
                         pack_bf16(o[8 * u + 6] * inv, o[8 * u + 7] * inv));
        fence_proxy_async_smem();
        mbar_arrive(&s.o_staged);
        // (after an abort the store is skipped; the warp leaves at its next wait)
        if (threadIdx.x == 256 && wait_or_abort(s, &s.o_staged, i & 1, p.err)) {
          tma_store_3d(&o_map, q_buf + ob * kQBytes, 0, g * grp, zrow);
          tma_store_3d(&o_map, q_buf + ob * kQBytes + kQBytes / 2, 64, g * grp, zrow);
          bulk_commit_group();
          bulk_wait_read_all();  // the buffer is read: Q of the tile two ahead may land
          mbar_arrive(&s.q_empty[ob]);
        }
      }
      if (warp == 8 && i + 2 < n_items) {
        // the softmax is done with slot ob's masks: they become those of tile i + 2
        if (!__all_sync(0xffffffffu, wait_or_abort(s, &s.info_free[ob], (i >> 1) & 1, p.err))) break;
        fill_masks(i + 2);
        mbar_arrive(&s.info_full[ob]);
      }
    }
    if (!kOutF32 && threadIdx.x == 256) bulk_wait_all();  // the output stores are complete
  }

  __syncthreads();
  if ((warp == 0 || warp == 6) && lane == 0 && s.abort) {
    // let the copies still in flight (at most the last ring's worth issued) land before
    // the CTA's shared memory is released
    const int nst = warp == 0 ? kKStages : kVStages;
    uint64_t* fullb = warp == 0 ? s.kfull : s.vfull;
    for (int n = issued > nst ? issued - nst : 0; n < issued; ++n)
      mbar_wait_bounded(&fullb[n % nst], (n / nst) & 1, kWaitLimit);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---- host side -----------------------------------------------------------------------
bool encode_kv(const Dev& p, int box_rows, CUtensorMap* out) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cuuint64_t(p.D), cuuint64_t(int64_t(p.b) * p.L * p.Hkv * 2 * p.R)};
  const cuuint64_t strides[1] = {cuuint64_t(p.D) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
  const cuuint32_t es[2] = {1, 1};
  return fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.kv, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_q(const Dev& p, int lcount, const void* q, CUtensorMap* out) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int grp = p.Hq / p.Hkv;
  const cuuint64_t dims[3] = {cuuint64_t(p.D), cuuint64_t(p.Hq), cuuint64_t(int64_t(p.b) * lcount * p.B)};
  const cuuint64_t strides[2] = {cuuint64_t(p.D) * 2, cuuint64_t(p.Hq) * p.D * 2};
  const cuuint32_t box[3] = {64, cuuint32_t(grp), cuuint32_t(p.B)};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_supported(const Dev& p) {
  const int grp = p.Hq / p.Hkv;
  return p.dtype == LS_BF16 && p.D == 128 && grp * p.B == 64 && p.R + 1 <= kMaxChunks * kChunk;
}

int tc_prepare(const Dev& p, TcPlan* plan) {
  static_assert(sizeof(CUtensorMap) <= sizeof(plan->kv_map), "tensor map size");
  plan->n_chunks = p.R / kChunk + 1;
  plan->tail_rows = p.R % kChunk;
  if (!encode_kv(p, kChunk, reinterpret_cast<CUtensorMap*>(plan->kv_map))) return LS_ERR_CUDA;
  if (plan->tail_rows > 0 && !encode_kv(p, plan->tail_rows, reinterpret_cast<CUtensorMap*>(plan->kv_tail_map)))
    return LS_ERR_CUDA;
  if (cudaFuncSetAttribute(attend_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
          cudaSuccess ||
      cudaFuncSetAttribute(attend_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
          cudaSuccess)
    return LS_ERR_CUDA;
  return LS_OK;
}

cudaError_t launch_attend_tc(const Dev& p, const TcPlan& plan, int lb, int lcount, const void* q,
                             const void* bk, const void* bv, int64_t bstride, float scale, int views,
                             void* out, int sms, AttendLaunch mode, bool side_by_side, cudaStream_t stream) {
  // Q in, and a bf16 O out, are [b, lcount, B, Hq, D]: one tile is the box (64 columns,
  // the group's heads, the block's queries) at (0 or 64, g * group, first query)
  CUtensorMap qmap, omap;
  if (!encode_q(p, lcount, q, &qmap)) return cudaErrorInvalidValue;
  if (p.out_f32)
    omap = qmap;  // unused: fp32 output is stored directly
  else if (!encode_q(p, lcount, out, &omap))
    return cudaErrorInvalidValue;
  TcArgs a{};
  a.lb = lb;
  a.lcount = lcount;
  a.n_tiles = p.b * lcount * p.Hkv;
  a.n_chunks = plan.n_chunks;
  a.tail_rows = plan.tail_rows;
  a.bk = static_cast<const __nv_bfloat16*>(bk);
  a.bv = static_cast<const __nv_bfloat16*>(bv);
  a.bstride = bstride;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = out;
  a.mode = mode;
  // chunks holding rows of a view that takes part are streamed; the last chunk always is
  // (it carries the boundary row), its arena rows only when a view needs them
  a.views = views;
  const bool win = (views & LS_VIEW_WINDOW) != 0, sum = (views & LS_VIEW_SUMMARY) != 0;
  for (int c = 0; c < plan.n_chunks; ++c) {
    const int lo = c * kChunk, hi = lo + kChunk < p.R ? lo + kChunk : p.R;  // arena rows [lo, hi)
    const bool need = (win && lo < p.W) || (sum && hi > (lo > p.W ? lo : p.W));
    if (c == plan.n_chunks - 1) {
      a.chunk_mask |= 1u << c;
      a.tail_load = need ? 1 : 0;
    } else if (need) {
      a.chunk_mask |= 1u << c;
    }
  }
  // at most one CTA per SM, tiles round robin, and no more CTAs than needed for the
  // fewest tiles per CTA: every CTA then gets the same number of tiles (512 tiles on 148
  // SMs: 128 CTAs x 4 instead of 68 x 4 + 80 x 3). The stream is bandwidth-bound, so the
  // idle SMs cost nothing while the ragged last wave would have.
  // Launches chained without waits (side_by_side) and of at most one wave take at most
  // half of the SMs (as few CTAs as the fewest tiles per CTA allows): the next layer's
  // launch is then resident beside this one and streams while this one drains, instead of
  // each SM starting a CTA per layer after the previous layer's CTA has left it (per-layer
  // calls, 4 layers after an L2 flush: 43.9 against 54.3 us).
  const int slots = (side_by_side && a.n_tiles <= sms) ? sms / 2 : sms;
  const int waves = (a.n_tiles + slots - 1) / slots;
  const int grid = (a.n_tiles + waves - 1) / waves;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  // scheduled once the kernel before it on `stream` triggers or completes (see AttendLaunch)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const CUtensorMap& kv = *reinterpret_cast<const CUtensorMap*>(plan.kv_map);
  const CUtensorMap& kv_tail = *reinterpret_cast<const CUtensorMap*>(plan.kv_tail_map);
  return p.out_f32 ? cudaLaunchKernelEx(&cfg, attend_tc_kernel<true>, p, a, kv, kv_tail, qmap, omap)
                   : cudaLaunchKernelEx(&cfg, attend_tc_kernel<false>, p, a, kv, kv_tail, qmap, omap);
}

}  // namespace ls
