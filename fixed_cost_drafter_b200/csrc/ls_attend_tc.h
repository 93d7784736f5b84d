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
// The kernel is always launched as the programmatic dependent of the kernel before it on
// `stream`: its threads wait on the device (griddepcontrol.wait) before they read what that
// kernel may write, and trigger their own dependents right after that wait. What may be
// read before the wait depends on what the caller knows about the kernel before it:
enum AttendLaunch : int {
  kAttendPlain = 0,        // nothing: every input after the wait
  kAttendAfterCommit = 1,  // the first tile's Q before the wait: an input complete before
                           // that kernel started (it is this state's commit kernel, or the
                           // caller says so with LS_ATTEND_INPUTS_READY)
  kAttendViewsSettled = 2, // no call has written the views since an attention launched on
                           // this stream: the first K/V chunks of the views before the wait
                           // (Q and the boundary rows after it)
  kAttendFree = 3          // settled views, and the caller's inputs were complete before the
                           // kernel before it started (LS_ATTEND_INPUTS_READY): no wait
};
// views: non-zero OR of LS_VIEW_* (the views that take part in the softmax).
// side_by_side: the caller chains launches that need not wait for one another
// (LS_ATTEND_INPUTS_READY): a launch of at most one wave of tiles then takes at most half
// of the SMs, so that the next launch's CTAs stream beside it.
cudaError_t launch_attend_tc(const Dev& p, const TcPlan& plan, int lb, int lcount, const void* q,
                             const void* bk, const void* bv, int64_t bstride, float scale, int views,
                             void* out, int sms, AttendLaunch mode, bool side_by_side, cudaStream_t stream);

}  // namespace ls
