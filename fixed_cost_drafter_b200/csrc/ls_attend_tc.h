// tcgen05 tensor-core path of the drafter block attention (sm_100a).
#pragma once
#include "ls_common.cuh"

namespace ls {

// Per-state constants of the tensor-core path: tensor maps over the arena's K/V rows
// (128-row chunks, and the shorter last chunk of each tile).
struct alignas(64) TcPlan {
  alignas(64) unsigned char kv_map[128];       // CUtensorMap, box 64 x 128 rows
  alignas(64) unsigned char kv_tail_map[128];  // CUtensorMap, box 64 x tail_rows (if tail_rows > 0)
  int32_t n_chunks;                             // 128-row chunks per tile: floor(R / 128) + 1
  int32_t tail_rows;                            // R mod 128: arena rows of the last chunk
};

bool tc_supported(const Dev& p);
int tc_prepare(const Dev& p, TcPlan* plan);
// after_commit: launched right behind ls_commit_round's kernel on the same stream as its
// programmatic dependent (the kernel waits on the device for the commit's writes).
// views: non-zero OR of LS_VIEW_* (the views that take part in the softmax).
cudaError_t launch_attend_tc(const Dev& p, const TcPlan& plan, int lb, int lcount, const void* q,
                             const void* bk, const void* bv, int64_t bstride, float scale, int views,
                             void* out, int sms, bool after_commit, cudaStream_t stream);

}  // namespace ls
