// Shared definitions of the LongSpark drafting-round kernels (sm_100a).
// State layout, slot validity, element conversion and the PTX wrappers used by the
// bulk-copy pipelines and the tcgen05 attention kernel.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/longspark.h"

namespace ls {

constexpr int kMaxScales = LS_MAX_SCALES;

// Device-side view of one drafting state: shapes plus region pointers in the arena.
struct Dev {
  int32_t b, L, Hkv, Hq, D, hidden, B, W, nsc, slots, R, dtype;
  int32_t out_f32;  // attention output in fp32 instead of dtype
  int32_t scales[kMaxScales];
  int64_t* counters;  // [b][L][1+nsc]
  int32_t* err;       // device error word
  int32_t* arrive;    // [b][L] arrivals of the (sequence, layer)'s KV-head CTAs in a commit
  char* kv;           // [b][L][Hkv][2][R][D] elements
  float* seg;         // [b][L][Hkv][nsc][slots][2][D]
  float* part;        // [b][L][Hkv][nsc][2][D]
  float* glob;        // [b][L][Hkv][2][D]
  char* boundary;     // [b][L][hidden] elements
  int32_t* samp_count;  // [b] arrivals of a sequence's CTAs in ls_accept_sampled
  float* samp_part;     // [b][kSampleMaxChunks] vocabulary chunk sums of ls_accept_sampled
  float* samp_seg;      // [b][kSampleMaxChunks][64] the chunks' segment sums (128 entries each)
  float* pro_part;      // [kProMaxSlots][128][boundary rows] split-tile partial sums of ls_draft_prologue
  int32_t* pro_count;   // [kProMaxGrid] arrivals of a split tile's pieces
};

constexpr int kSampleChunk = 8192;     // vocabulary entries per CTA of ls_accept_sampled
constexpr int kSampleMaxChunks = 64;   // vocab <= 524288

// ls_draft_prologue: at most this many CTAs (one per SM), tiles of 128 weight rows, 64
// hidden entries per k-step, at most 256 activation rows per tile.
constexpr int kProMaxGrid = 160;
constexpr int kProTileN = 128;
constexpr int kProKStep = 64;
constexpr int kProMaxAct = 256;

__host__ __device__ inline bool prologue_shapes_ok(int dtype, int hidden, int Hq, int Hkv, int D, int B) {
  return dtype == LS_BF16 && hidden % kProKStep == 0 && (Hq * D) % kProTileN == 0 && (2 * Hkv * D) % kProTileN == 0 &&
         B <= kProMaxAct;
}
// MMA N of the boundary projection: the batch (at most 256 per tile) rounded up to 16.
__host__ __device__ inline int prologue_boundary_rows(int batch) {
  const int r = batch < kProMaxAct ? batch : kProMaxAct;
  return (r + 15) & ~15;
}
// Split pieces of boundary tiles at most in flight (a CTA's range of k-steps touches at
// most one more tile than it finishes): 2 per CTA.
constexpr int kProMaxSlots = 2 * kProMaxGrid;

__host__ __device__ inline int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

// Arena layout for a validated config (host and device agree by construction).
struct Layout {
  int64_t counters, error, sync, kv, seg, part, glob, boundary, sample, prologue, total;
  int32_t R, elem;
};

__host__ inline Layout make_layout(const ls_config& c) {
  Layout y{};
  y.elem = c.dtype == LS_BF16 ? 2 : 4;
  y.R = c.window + c.n_scales * (c.slots_per_scale + 1) + 1;
  const int64_t tiles = int64_t(c.batch) * c.n_layers * c.n_kv_heads;
  int64_t off = 0;
  y.counters = off; off = align256(off + int64_t(c.batch) * c.n_layers * (1 + c.n_scales) * 8);
  y.error = off;    off = align256(off + 16);
  y.sync = off;     off = align256(off + int64_t(c.batch) * c.n_layers * 4);
  y.kv = off;       off = align256(off + tiles * 2 * y.R * c.head_dim * y.elem);
  y.seg = off;      off = align256(off + tiles * c.n_scales * c.slots_per_scale * 2 * c.head_dim * 4);
  y.part = off;     off = align256(off + tiles * c.n_scales * 2 * c.head_dim * 4);
  y.glob = off;     off = align256(off + tiles * 2 * c.head_dim * 4);
  y.boundary = off; off = align256(off + int64_t(c.batch) * c.n_layers * c.hidden * y.elem);
  y.sample = off;   off = align256(off + int64_t(c.batch) * (1 + kSampleMaxChunks + kSampleMaxChunks * 64) * 4);
  y.prologue = off;
  if (prologue_shapes_ok(c.dtype, c.hidden, c.n_q_heads, c.n_kv_heads, c.head_dim, c.block))
    off = align256(off + int64_t(kProMaxSlots) * kProTileN * prologue_boundary_rows(c.batch) * 4 + kProMaxGrid * 4);
  y.total = off;
  return y;
}

// ---- element conversion -------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kVec = 4;  // elements per 16-byte vector
  __device__ static inline void to_f32(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  __device__ static inline uint4 from_f32(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
  __device__ static inline float load1(const void* p, int64_t i) {
    return reinterpret_cast<const float*>(p)[i];
  }
  __device__ static inline void store1(void* p, int64_t i, float x) {
    reinterpret_cast<float*>(p)[i] = x;
  }
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kVec = 8;
  __device__ static inline void to_f32(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ static inline uint4 from_f32(const float* f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);  // RNE
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
  __device__ static inline float load1(const void* p, int64_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  }
  __device__ static inline void store1(void* p, int64_t i, float x) {
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
  }
};

// ---- slot validity of the arena rows of one tile --------------------------------
// Row r < W: ring slot r, filled once len > r. Then per scale k: slots 0..slots-1
// (filled once n_seg[k] > i) and the partial mean (non-empty when len - n_seg*s > 0).
// Last row: the global mean (len > 0).
__device__ inline bool arena_row_valid(const Dev& p, int r, int64_t len, const int64_t* nseg) {
  if (r < p.W) return r < len;
  int rr = r - p.W;
  const int per = p.slots + 1;
  int k = rr / per;
  if (k >= p.nsc) return len > 0;  // global mean row
  int i = rr - k * per;
  if (i < p.slots) return i < nseg[k];
  return len - nseg[k] * int64_t(p.scales[k]) > 0;
}

__device__ inline void set_err(int32_t* err, int32_t bits) { atomicOr(err, bits); }

// ---- mbarrier / bulk-copy PTX ---------------------------------------------------
__device__ inline uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ inline void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ inline void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ inline bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: gives up after `limit` polls (each poll itself suspends for a
// hardware-chosen interval) and reports false, so no kernel can spin forever.
__device__ inline bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
constexpr uint32_t kWaitLimit = 1u << 22;

// Programmatic dependent launch. A kernel launched with the programmatic-serialization
// attribute may start while the kernel before it on the stream still runs; its threads
// call grid_dependency_wait() before they read anything that kernel writes (the wait
// returns once that grid has completed and its writes are visible; without the launch
// attribute it returns at once). The earlier kernel calls allow_dependent_launch() to let
// the dependent be scheduled before it completes.
__device__ inline void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void allow_dependent_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Bulk asynchronous global->shared copy on the TMA engine (no tensor map, into this CTA only).
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ inline void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ inline void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ inline uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ---- paged KV cache ---------------------------------------------------------------
// paged_row: byte address of the row (all KV heads) at position `pos` of sequence b in the
// layer whose pages start at `base`: page block_table[b][pos / page_size], offset
// pos mod page_size. A position past the block table or a page id outside
// [0, num_pages) sets LS_DEVERR_PAGE and gives the same offset in page 0, so no access
// leaves the caller's pages. Its three steps, for callers that look pages up ahead:
// Page index and in-page offset of position `pos`.
__device__ inline int64_t paged_index(const ls_paged_kv& kv, int64_t pos, int& off) {
  const int ps = kv.page_size;
  if ((ps & (ps - 1)) == 0) {  // the usual page sizes: shift and mask
    off = int(pos & (ps - 1));
    return pos >> (__ffs(ps) - 1);
  }
  if (pos < (int64_t(1) << 32)) {
    const uint32_t q = uint32_t(pos) / uint32_t(ps);
    off = int(uint32_t(pos) - q * uint32_t(ps));
    return q;
  }
  const int64_t pi = pos / ps;
  off = int(pos - pi * ps);
  return pi;
}
// The block table's entry for page index pi of sequence b (-1 past the table). The load is
// issued here; a caller that uses the value later overlaps its latency with other work.
__device__ inline int32_t paged_entry(const ls_paged_kv& kv, int b, int64_t pi) {
  return pi < kv.max_blocks ? __ldg(kv.block_table + int64_t(b) * kv.max_blocks + pi) : -1;
}
// Byte address of offset `off` in page `entry` of the layer at `base`; an entry outside
// [0, num_pages) sets LS_DEVERR_PAGE and gives the same offset in page 0.
__device__ inline const char* paged_at(const ls_paged_kv& kv, const char* base, int32_t entry, int off, int elem,
                                       int32_t* err) {
  int64_t page = entry;
  if (page < 0 || page >= kv.num_pages) {
    set_err(err, LS_DEVERR_PAGE);
    page = 0;
  }
  return base + (page * kv.page_stride + int64_t(off) * kv.slot_stride) * elem;
}
__device__ inline const char* paged_row(const ls_paged_kv& kv, const char* base, int b, int64_t pos, int elem,
                                        int32_t* err) {
  int off;
  const int64_t pi = paged_index(kv, pos, off);
  return paged_at(kv, base, paged_entry(kv, b, pi), off, elem, err);
}

// Byte address of slot `slot` (page * page_size + offset) in the layer at `base`; a slot
// outside the pool sets LS_DEVERR_PAGE and gives slot 0.
__device__ inline const char* paged_slot(const ls_paged_kv& kv, const char* base, int64_t slot, int elem,
                                         int32_t* err) {
  const int ps = kv.page_size;
  int64_t page;
  int off;
  if ((ps & (ps - 1)) == 0) {
    page = slot >> (__ffs(ps) - 1);
    off = int(slot & (ps - 1));
  } else {
    page = slot / ps;
    off = int(slot - page * ps);
  }
  if (slot < 0 || page >= kv.num_pages) {
    set_err(err, LS_DEVERR_PAGE);
    page = 0;
    off = 0;
  }
  return base + (page * kv.page_stride + int64_t(off) * kv.slot_stride) * elem;
}

}  // namespace ls
