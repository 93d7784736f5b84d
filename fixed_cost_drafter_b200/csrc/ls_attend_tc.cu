// Drafter block attention over the three views on the 5th-generation tensor cores:
// LongSpark paper page, Figure 2 caption (c): the drafter attends over fixed-size views,
// so its cost does not depend on the prefix length.
//
// One tile = (sequence, layer, KV head g): M = (Hq/Hkv) * B = 64 query rows (the GQA
// group's heads x the block's queries, row m = i * group + j) against the tile's
// kv_rows <= 768 arena rows (ring window + summary mean rows) plus the boundary row.
// Because the views are fixed-size, the whole score matrix S = Q K^T of a tile fits in
// tensor memory at once, so the softmax is exact (global row max first, then one pass of
// exponentials) and the output accumulator is never rescaled.
//
// Persistent kernel, one CTA per SM, 6 warps:
//   warp 0    TMA producer: Q of each tile through a 3-D tensor map (two 64-column
//             swizzled halves), then the tile's K rows and V rows in chunks of 128 rows
//             through a ring of shared-memory stages (tensor map over the state arena).
//   warp 1    TMEM allocator and the single MMA-issuing thread: tcgen05.mma kind::f16
//             (bf16 in, fp32 accumulate), M = 64. S chunk c goes to TMEM columns
//             128*(c/2) at lane offset 16*(c%2) (the M = 64 accumulator fills lanes 0-15
//             of each 32-lane subpartition; the odd chunk uses lanes 16-31). O (64 x 128
//             fp32) sits in columns 384..511.
//   warps 2-5 softmax and epilogue, one TMEM subpartition each: per row the boundary
//             logit on CUDA cores, row max over all chunks, exp2, bf16 P written to shared
//             memory in the MMA's swizzled K-major layout; after P V, the boundary value's
//             share, 1/rowsum, bf16 output.
// Every wait is bounded; a wait that runs out sets LS_DEVERR_WAIT_TIMEOUT and the CTA
// stops, lets its issued copies land, frees its tensor memory and returns.
#include <cuda.h>

#include "ls_attend_tc.h"

namespace ls {

namespace {

constexpr int kStages = 4;
constexpr int kChunk = 128;            // arena rows per chunk
constexpr int kMaxChunks = 6;          // kv_rows <= 768
constexpr int kThreads = 192;
constexpr int kQBytes = 64 * 128 * 2;  // one Q tile (two 8 KB halves)
constexpr int kPBytes = 64 * 128 * 2;  // one P chunk (two 8 KB halves)
constexpr int kStageBytes = kChunk * 128 * 2;  // one K or V chunk (two 16 KB halves)
constexpr int kSmemBytes = 2 * kQBytes + 2 * kPBytes + kStages * kStageBytes + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 384;

struct TcArgs {
  int32_t lb, lcount, n_tiles, n_chunks, tail_rows;
  const __nv_bfloat16* bk;
  const __nv_bfloat16* bv;
  int64_t bstride;
  float scale_log2;  // softmax_scale * log2(e)
  void* out;         // bf16, or fp32 when Dev::out_f32
};

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t s_full, s_free, o_full, o_empty;
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t vmask[kMaxChunks * kChunk / 32];
};

// ---- PTX wrappers -------------------------------------------------------------------
__device__ inline void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ inline void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ inline void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
//   K-major operand: 8-row x 128-byte atoms, SBO = 1024 B between 8-row groups.
//   MN-major operand: 8 K-rows x 64 elements per atom, SBO = 1024 B between 8-row K groups,
//   LBO = distance to the next 64-element block along MN.
__device__ inline uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((addr >> 4) & 0x3FFF);
  d |= uint64_t((lbo >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;  // descriptor version for sm_100
  d |= uint64_t(2) << 61;  // 128-byte swizzle
  return d;
}
// Instruction descriptor: kind::f16 with bf16 A/B, fp32 D, M = 64.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn_major) {
  return (1u << 4)      // D fp32
         | (1u << 7)    // A bf16
         | (1u << 10)   // B bf16
         | (uint32_t(b_mn_major) << 16)
         | (uint32_t(n >> 3) << 17)
         | (uint32_t(64 >> 4) << 24);
}
__device__ inline void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ inline void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ inline void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ inline void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ inline void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ inline float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ inline void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ inline uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Bounded wait that also gives up when another role has already aborted.
__device__ inline bool wait_or_abort(Bars& s, uint64_t* bar, uint32_t parity, int32_t* err) {
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

__global__ void __launch_bounds__(kThreads, 1)
attend_tc_kernel(const Dev p, const TcArgs a, const __grid_constant__ CUtensorMap kv_map,
                 const __grid_constant__ CUtensorMap kv_tail_map, const __grid_constant__ CUtensorMap q_map) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ Bars s;
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_buf = smem;                           // [2][kQBytes]
  unsigned char* p_buf = q_buf + 2 * kQBytes;            // [2][kPBytes]
  unsigned char* st_buf = p_buf + 2 * kPBytes;           // [kStages][kStageBytes]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nC = a.n_chunks;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&s.full[i], 1); mbar_init(&s.empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.q_full[i], 1); mbar_init(&s.q_empty[i], 2);
      mbar_init(&s.p_full[i], 1); mbar_init(&s.p_empty[i], 1);
    }
    mbar_init(&s.s_full, 1); mbar_init(&s.s_free, 1);
    mbar_init(&s.o_full, 1); mbar_init(&s.o_empty, 1);
    s.abort = 0;
    fence_mbar_init();
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

  int issued_stages = 0, landed_stages = 0;  // producer bookkeeping for the drain

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_map(&kv_map); prefetch_map(&kv_tail_map); prefetch_map(&q_map);
      int st = 0, it = 0;
      for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++it) {
        int b, lc, g;
        tile_coords(t, p, a.lcount, b, lc, g);
        const int qb = it & 1;
        if (!wait_or_abort(s, &s.q_empty[qb], ((it >> 1) & 1) ^ 1, p.err)) break;
        mbar_arrive_expect_tx(&s.q_full[qb], kQBytes);
        const int grp = p.Hq / p.Hkv;
        const int zrow = (b * a.lcount + lc) * p.B;
        tma_load_3d(q_buf + qb * kQBytes, &q_map, 0, g * grp, zrow, &s.q_full[qb]);
        tma_load_3d(q_buf + qb * kQBytes + kQBytes / 2, &q_map, 64, g * grp, zrow, &s.q_full[qb]);
        const int l = a.lb + lc;
        const int64_t tile = (int64_t(b) * p.L + l) * p.Hkv + g;
        bool ok = true;
        for (int t2 = 0; t2 < 2 && ok; ++t2) {
          for (int c = 0; c < nC; ++c, ++st) {
            const int sidx = st % kStages;
            if (!wait_or_abort(s, &s.empty[sidx], ((st / kStages) & 1) ^ 1, p.err)) { ok = false; break; }
            const bool tail = c == nC - 1;
            const int rows = tail ? a.tail_rows : kChunk;
            mbar_arrive_expect_tx(&s.full[sidx], uint32_t(rows * 256));
            const int y = int((tile * 2 + t2) * p.R + int64_t(c) * kChunk);
            unsigned char* dst = st_buf + sidx * kStageBytes;
            const CUtensorMap* m = tail ? &kv_tail_map : &kv_map;
            tma_load_2d(dst, m, 0, y, &s.full[sidx]);
            tma_load_2d(dst + kStageBytes / 2, m, 64, y, &s.full[sidx]);
            ++issued_stages;
          }
        }
        if (!ok) break;
      }
      landed_stages = st;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int st = 0, it = 0, pu[2] = {0, 0};
      const uint32_t q_base = smem_u32(q_buf), p_base = smem_u32(p_buf), s_base = smem_u32(st_buf);
      const uint32_t id_qk_full = idesc_bf16(kChunk, false);
      const uint32_t id_qk_tail = idesc_bf16(a.tail_rows, false);
      const uint32_t id_pv = idesc_bf16(128, true);
      bool ok = true;
      for (int t = blockIdx.x; t < a.n_tiles && ok; t += gridDim.x, ++it) {
        const int qb = it & 1;
        if (!wait_or_abort(s, &s.q_full[qb], (it >> 1) & 1, p.err)) break;
        if (!wait_or_abort(s, &s.s_free, (it & 1) ^ 1, p.err)) break;
        tc_fence_after();
        // S = Q K^T, chunk by chunk
        for (int c = 0; c < nC; ++c, ++st) {
          const int sidx = st % kStages;
          if (!wait_or_abort(s, &s.full[sidx], (st / kStages) & 1, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t(16 * (c & 1)) << 16) + uint32_t(128 * (c >> 1));
          const uint32_t idesc = c == nC - 1 ? id_qk_tail : id_qk_full;
          const uint32_t kb = s_base + sidx * kStageBytes;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * (kQBytes / 2) + (k & 3) * 32;
            const uint32_t koff = (k >> 2) * (kStageBytes / 2) + (k & 3) * 32;
            mma_bf16(d, sdesc(q_base + qb * kQBytes + off, 16, 1024), sdesc(kb + koff, 16, 1024), idesc,
                     k > 0);
          }
          mma_commit(&s.empty[sidx]);
        }
        if (!ok) break;
        mma_commit(&s.q_empty[qb]);
        mma_commit(&s.s_full);
        // O = P V, chunk by chunk, once the softmax has written P_c
        if (!wait_or_abort(s, &s.o_empty, (it & 1) ^ 1, p.err)) break;
        for (int c = 0; c < nC; ++c, ++st) {
          const int sidx = st % kStages;
          const int pb = c & 1;
          if (!wait_or_abort(s, &s.full[sidx], (st / kStages) & 1, p.err)) { ok = false; break; }
          if (!wait_or_abort(s, &s.p_full[pb], pu[pb] & 1, p.err)) { ok = false; break; }
          ++pu[pb];
          tc_fence_after();
          const int rows = c == nC - 1 ? a.tail_rows : kChunk;
          const uint32_t vb = s_base + sidx * kStageBytes;
          for (int k = 0; k < rows / 16; ++k) {
            const uint32_t poff = (k >> 2) * (kPBytes / 2) + (k & 3) * 32;
            // V chunk: rows = keys (K dim), 128-byte rows per 64-column half: MN-major B,
            // LBO = distance to the second half, SBO = 8 rows.
            mma_bf16(tmem + kOCol, sdesc(p_base + pb * kPBytes + poff, 16, 1024),
                     sdesc(vb + k * 2048, kStageBytes / 2, 1024), id_pv, (c > 0 || k > 0));
          }
          mma_commit(&s.empty[sidx]);
          mma_commit(&s.p_empty[pb]);
        }
        if (!ok) break;
        mma_commit(&s.o_full);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // The four warps leave the tile loop only together, right after a named barrier,
    // when the shared abort flag is set (a wait that ran out sets it before the barrier).
    const int sw = warp - 2;            // 0..3
    const int sub = warp & 3;           // TMEM subpartition this warp may access
    const int half = lane >> 4;         // 0: even chunks, 1: odd chunks
    const int row = 16 * sub + (lane & 15);
    const uint32_t trow = tmem + (uint32_t(32 * sub) << 16);
    const int grp = p.Hq / p.Hkv;
    const int tid = sw * 32 + lane;     // 0..127
    const int ncb = (nC + 1) >> 1;
    volatile uint32_t* abort_flag = &s.abort;
    auto group_sync_ok = [&]() {
      named_sync(1, 128);
      return *abort_flag == 0;
    };
    int it = 0, pu[2] = {0, 0};
    for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++it) {
      int b, lc, g;
      tile_coords(t, p, a.lcount, b, lc, g);
      const int l = a.lb + lc;
      const int qb = it & 1;
      // validity of the tile's arena rows as a bit mask
      {
        const int64_t* ctr = p.counters + (int64_t(b) * p.L + l) * (1 + p.nsc);
        const int64_t len = ctr[0];
        int64_t nseg[kMaxScales];
#pragma unroll
        for (int k = 0; k < kMaxScales; ++k) nseg[k] = k < p.nsc ? ctr[1 + k] : 0;
        for (int base = 0; base < nC * kChunk; base += 128) {
          const int r = base + tid;
          const bool v = r < p.R && arena_row_valid(p, r, len, nseg);
          const unsigned bal = __ballot_sync(0xffffffffu, v);
          if (lane == 0) s.vmask[(base >> 5) + sw] = bal;
        }
      }
      // boundary logit on CUDA cores: q_row . boundary_k (each half of the pair does 64 d)
      const bool q_ok = wait_or_abort(s, &s.q_full[qb], (it >> 1) & 1, p.err);
      float blog = 0.f;
      const int64_t boff = (int64_t(b) * p.L + l) * a.bstride + int64_t(g) * 128;
      if (q_ok) {
        const unsigned char* qrow = q_buf + qb * kQBytes + half * (kQBytes / 2) + row * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 qv = *reinterpret_cast<const uint4*>(qrow + ((ch ^ (row & 7)) << 4));
          const uint4 kv4 = ld_nc_v4(a.bk + boff + half * 64 + ch * 8);
          float qf[8], kf[8];
          Elem<__nv_bfloat16>::to_f32(qv, qf);
          Elem<__nv_bfloat16>::to_f32(kv4, kf);
#pragma unroll
          for (int e = 0; e < 8; ++e) blog = fmaf(qf[e], kf[e], blog);
        }
      }
      blog += __shfl_xor_sync(0xffffffffu, blog, 16);
      if (!group_sync_ok()) break;
      if (tid == 0) mbar_arrive(&s.q_empty[qb]);

      // all S chunks of this tile are in TMEM: row max over every valid slot
      const bool s_ok = wait_or_abort(s, &s.s_full, it & 1, p.err);
      tc_fence_after();
      float mx = -INFINITY;
      if (__all_sync(0xffffffffu, s_ok)) {
        for (int cb = 0; cb < ncb; ++cb) {
          const int c = 2 * cb + half;
#pragma unroll 1
          for (int q4 = 0; q4 < 4; ++q4) {
            float v[32];
            tmem_ld32(trow + uint32_t(cb * 128 + q4 * 32), v);
            const uint32_t m = c < nC ? s.vmask[(c * kChunk + q4 * 32) >> 5] : 0u;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if ((m >> j) & 1u) mx = fmaxf(mx, v[j]);
          }
        }
      }
      if (!group_sync_ok()) break;
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      mx = fmaxf(mx, blog);
      const float mscaled = mx * a.scale_log2;
      // exponentials, row sums, bf16 P into the swizzled K-major tile of its chunk
      float sum = 0.f;
      bool aborted = false;
      for (int cb = 0; cb < ncb; ++cb) {
        const int c = 2 * cb + half;
        const bool mine = c < nC;
        const bool pe_ok = !mine || wait_or_abort(s, &s.p_empty[half], (pu[half] & 1) ^ 1, p.err);
        const bool go = __all_sync(0xffffffffu, pe_ok);
        unsigned char* prow = p_buf + half * kPBytes + row * 128;
#pragma unroll 1
        for (int q4 = 0; q4 < 4 && go; ++q4) {
          float v[32];
          tmem_ld32(trow + uint32_t(cb * 128 + q4 * 32), v);
          if (!mine) continue;
          const uint32_t m = s.vmask[(c * kChunk + q4 * 32) >> 5];
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float p0 = ((m >> j) & 1u) ? ex2(fmaf(v[j], a.scale_log2, -mscaled)) : 0.f;
            const float p1 = ((m >> (j + 1)) & 1u) ? ex2(fmaf(v[j + 1], a.scale_log2, -mscaled)) : 0.f;
            sum += p0 + p1;
            pk[j >> 1] = pack_bf16(p0, p1);
          }
          // keys q4*32 .. q4*32+31 of this chunk: half (q4 >> 1) of the P tile, 16-byte
          // pieces (q4 & 1)*4 .. +3 of the row, swizzled by the row's position in its atom
          unsigned char* dst = prow + (q4 >> 1) * (kPBytes / 2);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int piece = (q4 & 1) * 4 + u;
            *reinterpret_cast<uint4*>(dst + ((piece ^ (row & 7)) << 4)) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          }
        }
        fence_proxy_async_smem();
        if (!group_sync_ok()) { aborted = true; break; }
        if (tid == 0) {
          mbar_arrive(&s.p_full[0]);
          if (2 * cb + 1 < nC) mbar_arrive(&s.p_full[1]);
        }
        if (2 * cb < nC) ++pu[0];
        if (2 * cb + 1 < nC) ++pu[1];
      }
      if (aborted) break;
      tc_fence_before();
      if (!group_sync_ok()) break;
      if (tid == 0) mbar_arrive(&s.s_free);
      sum += __shfl_xor_sync(0xffffffffu, sum, 16);
      const float pbd = ex2(fmaf(blog, a.scale_log2, -mscaled));
      sum += pbd;
      const float inv = 1.0f / sum;

      // epilogue: O row (lanes 0-15 of each subpartition) + boundary share, normalised
      const bool o_ok = wait_or_abort(s, &s.o_full, it & 1, p.err);
      tc_fence_after();
      const int i = row / grp, j = row - (row / grp) * grp;
      const int64_t orow = (((int64_t(b) * a.lcount + lc) * p.B + i) * p.Hq + g * grp + j) * 128;
      const bool o_go = __all_sync(0xffffffffu, o_ok);
#pragma unroll 1
      for (int q4 = 0; q4 < 4 && o_go; ++q4) {
        float v[32];
        tmem_ld32(trow + kOCol + uint32_t(q4 * 32), v);
        if (half == 0) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 bv4 = ld_nc_v4(a.bv + boff + q4 * 32 + u * 8);
            float bf[8];
            Elem<__nv_bfloat16>::to_f32(bv4, bf);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[u * 8 + e] = fmaf(pbd, bf[e], v[u * 8 + e]) * inv;
          }
          if (p.out_f32) {
            float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow + q4 * 32);
#pragma unroll
            for (int u = 0; u < 8; ++u) o4[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
          } else {
            uint4* o4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow + q4 * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              o4[u] = make_uint4(pack_bf16(v[8 * u], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
                                 pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
          }
        }
      }
      tc_fence_before();
      if (!group_sync_ok()) break;
      if (tid == 0) mbar_arrive(&s.o_empty);
    }
  }

  __syncthreads();
  if (warp == 0 && lane == 0 && s.abort) {
    // let the copies still in flight (at most the last kStages issued) land before the
    // CTA's shared memory is released
    for (int st = landed_stages > kStages ? landed_stages - kStages : 0; st < landed_stages; ++st)
      mbar_wait_bounded(&s.full[st % kStages], (st / kStages) & 1, kWaitLimit);
  }
  (void)issued_stages;
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---- host side -----------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

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
  return p.dtype == LS_BF16 && p.D == 128 && grp * p.B == 64 && p.R <= kMaxChunks * kChunk;
}

int tc_prepare(const Dev& p, TcPlan* plan) {
  static_assert(sizeof(CUtensorMap) <= sizeof(plan->kv_map), "tensor map size");
  plan->n_chunks = (p.R + kChunk - 1) / kChunk;
  const int tail = p.R - (plan->n_chunks - 1) * kChunk;
  plan->tail_rows = (tail + 15) / 16 * 16;
  if (!encode_kv(p, kChunk, reinterpret_cast<CUtensorMap*>(plan->kv_map))) return LS_ERR_CUDA;
  if (!encode_kv(p, plan->tail_rows, reinterpret_cast<CUtensorMap*>(plan->kv_tail_map))) return LS_ERR_CUDA;
  if (cudaFuncSetAttribute(attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return LS_ERR_CUDA;
  return LS_OK;
}

cudaError_t launch_attend_tc(const Dev& p, const TcPlan& plan, int lb, int lcount, const void* q,
                             const void* bk, const void* bv, int64_t bstride, float scale, void* out,
                             int sms, cudaStream_t stream) {
  CUtensorMap qmap;
  if (!encode_q(p, lcount, q, &qmap)) return cudaErrorInvalidValue;
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
  const int grid = a.n_tiles < sms ? a.n_tiles : sms;
  attend_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(
      p, a, *reinterpret_cast<const CUtensorMap*>(plan.kv_map),
      *reinterpret_cast<const CUtensorMap*>(plan.kv_tail_map), qmap);
  return cudaGetLastError();
}

}  // namespace ls
