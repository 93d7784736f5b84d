/*
 * longspark.h — C ABI of the LongSpark fixed-cost drafting round on B200 (sm_100a).
 *
 * Method: "LongSpark: Efficient speculative decoding with a fixed-cost parallel
 * drafter" (arXiv 2609.37029), as printed on the thelatestinai.com paper page:
 *   - Figure 2 caption: one decoding round = (a) the target verifies the proposed
 *     block, (b) three fixed-size context views are extracted from the target's
 *     state — a boundary state, a recent KV window and a global context summary —
 *     and (c) the drafter proposes the next block from those views at a cost that
 *     does not depend on the prefix length.
 *   - Figure 3 caption: the global summary is initialised over the whole prefix at
 *     target prefill and afterwards updated only from the newly retained KV rows N,
 *     with Delta = |N| <= B + 1.
 *   - Figure 1 caption / abstract: O(1) drafting cost and a drafter state whose size
 *     does not grow with the prefix ("fixed-size, multiscale views").
 * The pages print no formula for the views; the definitions used here are:
 *   accept scan   a = number of leading positions i < B with draft[i] == target[i];
 *                 next token = target[a]; Delta = a + 1 retained rows (verify rows 0..a).
 *   window        the last min(len, W) retained K/V rows; row p lives in ring slot p mod W.
 *   summary       per tapped layer and KV head, for each scale s_k: segment j covers the
 *                 absolute rows [j*s_k, (j+1)*s_k); the slots hold the K/V means of the
 *                 `slots` most recent complete segments (segment j in slot j mod slots),
 *                 plus the open partial segment (its sum; its mean is an attention slot),
 *                 plus one running mean over all retained rows.
 *   boundary      the tapped-layer hidden vectors at the last retained position.
 *   attention     per (layer, query head qh), KV head g = qh / (Hq/Hkv): softmax(q k^T * scale)
 *                 over [boundary, window rows, per scale: slots + partial mean, global mean],
 *                 empty slots masked, no mask among the B block queries.
 *
 * Conventions for every entry point:
 *   - Return value: LS_OK (0) or a negative LS_ERR_* code. Nothing traps or aborts.
 *   - Every d_* pointer is DEVICE memory owned by the caller; h_* pointers are host
 *     memory owned by the caller. The library never allocates device memory; the only
 *     host allocation is the opaque ls_state handle (ls_init_state / ls_destroy_state).
 *   - Device work is enqueued asynchronously on `stream`; no call synchronises except
 *     ls_read_state and ls_get_error, which say so.
 *   - Element types: `dtype` (LS_BF16 or LS_F32) is the type of K/V/hidden/q/out and of
 *     the window and mirror rows in the arena. Summary sums and segment means are fp32.
 *   - Kernels never trap. Conditions found on the device (bad prefix length, bounded
 *     waits that ran out) set bits in the device error word; read it with ls_get_error.
 *   - A state belongs to the device that was current at ls_init_state. Every call that
 *     takes a state returns LS_ERR_INVALID_ARG, and does nothing, while another device
 *     is current.
 */
#ifndef LONGSPARK_H_
#define LONGSPARK_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define LS_API __attribute__((visibility("default")))
#else
#define LS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------------ */
#define LS_OK                   0
#define LS_ERR_INVALID_ARG    (-1)  /* null pointer, negative size, bad enum           */
#define LS_ERR_SHAPE          (-2)  /* sizes inconsistent with each other or the arena  */
#define LS_ERR_UNSUPPORTED    (-3)  /* valid for the method, not for this GPU path      */
#define LS_ERR_CUDA           (-4)  /* a CUDA runtime call failed                       */
#define LS_ERR_DEVICE         (-5)  /* the device error word holds a non-zero code      */
#define LS_ERR_DEVICE_TIMEOUT (-6)  /* a bounded device wait gave up                    */
#define LS_ERR_SCRATCH_LIMIT  (-7)  /* ls_prefill_summary_noalloc: the chunk needs more
                                       than the library's fixed 16 MiB scratch        */

/* ---- device error word bits (ls_get_error) ----------------------------------- */
#define LS_DEVERR_PREFIX_LEN   0x1  /* prefix_len[b] < 0 or beyond what the buffers hold */
#define LS_DEVERR_WAIT_TIMEOUT 0x2  /* an mbarrier wait exceeded its iteration limit     */
#define LS_DEVERR_ORDER        0x4  /* prefill chunk does not continue the state          */
#define LS_DEVERR_SAMPLE       0x8  /* ls_accept_sampled: a draft id outside the vocabulary
                                       or a draw with no probability mass;
                                       ls_commit_accepted: a count outside [0, B]       */
#define LS_DEVERR_PAGE        0x10  /* paged calls: a position past the block table's
                                       max_blocks pages or a page id outside
                                       [0, num_pages) (the rows are read from page 0)  */

/* ---- views (Figure 2 caption (b); the component ablations of Table 5) -------- */
#define LS_VIEW_BOUNDARY 0x1        /* the boundary state (one key/value row)          */
#define LS_VIEW_WINDOW   0x2        /* the recent KV window (W ring rows)              */
#define LS_VIEW_SUMMARY  0x4        /* the global context summary (segment means per
                                       scale, partial means, global mean)             */
#define LS_VIEW_ALL      0x7
/* Launch hint for ls_draft_attend_views, OR-ed into `views`: the call's queries and
 * boundary rows were complete before the kernel launched just before this call on
 * `stream` started, and that kernel neither reads nor writes d_out (e.g. the drafter's
 * queries of every layer came from one earlier ls_draft_prologue, and the attention is
 * called layer by layer). The attention may then read those inputs, and write d_out,
 * while that kernel still runs, so consecutive per-layer calls overlap. A hint that
 * does not hold gives wrong outputs (never a fault).                                  */
#define LS_ATTEND_INPUTS_READY 0x100

/* ---- dtypes and flags -------------------------------------------------------- */
#define LS_F32  0
#define LS_BF16 1
#define LS_FLAG_FORCE_SIMT 0x1      /* run draft attention on CUDA cores even where the
                                       tcgen05 tensor-core kernel applies              */
#define LS_FLAG_OUT_F32    0x2      /* ls_draft_attend writes fp32 outputs (otherwise
                                       `dtype`); a bf16 output adds its own rounding of
                                       up to 2^-8 |out| to the attention's error       */

#define LS_MAX_SCALES 4

/* Shapes of one drafting state (one batch of sequences).
 *   batch b, n_layers L (tapped layers), n_kv_heads Hkv (<= 8), n_q_heads Hq (multiple of Hkv),
 *   head_dim D (multiple of 8, <= 256), hidden (multiple of 8), block B (1..32),
 *   window W (>= B+1), n_scales (1..4), scales ascending, each >= B+1,
 *   each dividing the next (so no segment of any scale straddles a larger one),
 *   slots_per_scale >= 1, dtype LS_F32 | LS_BF16, flags LS_FLAG_*.              */
typedef struct {
  int32_t batch, n_layers, n_kv_heads, n_q_heads, head_dim, hidden;
  int32_t block;
  int32_t window;
  int32_t n_scales;
  int32_t scales[LS_MAX_SCALES];
  int32_t slots_per_scale;
  int32_t dtype;
  int32_t flags;
} ls_config;

/* Byte offsets (from the arena base) and shapes of the regions of the state arena.
 * All offsets are multiples of 256. e = element size of `dtype`.
 *   counters  int64 [b][L][1 + n_scales]: retained length len, then for each scale the
 *             number of segments finalised so far (floor(len / s_k)).
 *   error     int32 [4]: word 0 is the device error word.
 *   sync      int32 [b][L]: zero between calls (arrival counts inside a commit).
 *   kv        e     [b][L][Hkv][2][kv_rows][D]: for K (index 0) and V (index 1) of each
 *             (sequence, layer, KV head) tile, rows 0..W-1 are the ring window, then for
 *             each scale k rows W + k*(slots+1) + i hold the mean of the segment in slot i
 *             (i < slots) or the open partial's mean (i == slots), and the last row
 *             (W + n_scales*(slots+1)) holds the global mean. kv_rows = that count + 1.
 *             These mean rows are the attention's copy, rounded to `dtype`.
 *   seg_mean  fp32  [b][L][Hkv][n_scales][slots][2][D]: segment means in full fp32.
 *   part_sum  fp32  [b][L][Hkv][n_scales][2][D]: sums of the open partial segments.
 *   glob_sum  fp32  [b][L][Hkv][2][D]: sum of all retained rows.
 *   boundary  e     [b][L][hidden]: hidden vectors at the last retained position.
 *   sample    int32 [b] then fp32 [b][64]: scratch of ls_accept_sampled (zero counts
 *             between calls), not part of any view.
 *   prologue  scratch of ls_draft_prologue (bf16 states whose shapes it supports; else
 *             empty): fp32 partial sums of the boundary projection's split tiles, then
 *             int32 arrival counts (zero between calls); not part of any view.         */
typedef struct {
  size_t total_bytes;
  size_t off_counters, off_error, off_sync, off_kv, off_seg_mean, off_part_sum, off_glob_sum,
         off_boundary;
  int32_t kv_rows;
  int32_t elem_bytes;
  size_t off_sample;
  size_t off_prologue;
} ls_layout;

typedef struct ls_state ls_state; /* opaque host handle */

/* A target's paged KV cache, read in place (an inference engine keeps K/V in fixed-size
 * pages; the views are extracted from that state, Figure 2 caption (b)). Host struct,
 * passed by pointer; the pointers in it are DEVICE memory owned by the caller.
 *   k_layers[l], v_layers[l]  base of tapped layer l's key / value pages (`dtype`), for
 *               l < n_layers (<= LS_MAX_PAGED_LAYERS); 16-byte aligned.
 *   Element (page, offset, h, d) of a layer sits at
 *               base[page * page_stride + offset * slot_stride + h * D + d]
 *               (e.g. pages [num_pages][page_size][Hkv][D]: slot_stride = Hkv*D,
 *               page_stride = page_size*Hkv*D; keys and values interleaved per page as
 *               [num_pages][2][page_size][Hkv][D]: page_stride = 2*page_size*Hkv*D and
 *               v_layers[l] = k_layers[l] + page_size*Hkv*D). Both strides are multiples
 *               of 8 elements, slot_stride >= Hkv*D.
 *   block_table int32 [b][max_blocks]: position p of sequence b is in page
 *               block_table[b][p / page_size] at offset p mod page_size.
 *   num_pages   page ids outside [0, num_pages) set LS_DEVERR_PAGE.
 *   verify_slots  NULL, or int64 [b][B+1]: the slot (page * page_size + offset) where the
 *               verify pass wrote verify row i of sequence b (an engine's slot mapping).
 *               The commit then reads the rows there instead of looking position len + i
 *               up in the block table, so its row loads no longer wait for that lookup.
 *               8-byte aligned; a slot outside the pool sets LS_DEVERR_PAGE. Prefill
 *               ignores it.
 * Each slot holds one row of all KV heads (a head-major page, [Hkv][page_size][D],
 * is not read).                                                                        */
#define LS_MAX_PAGED_LAYERS 64
typedef struct {
  const void* k_layers[LS_MAX_PAGED_LAYERS];
  const void* v_layers[LS_MAX_PAGED_LAYERS];
  int64_t page_stride;
  int64_t slot_stride;
  const int32_t* block_table;
  int32_t max_blocks;
  int32_t page_size;
  int64_t num_pages;
  const int64_t* verify_slots;
} ls_paged_kv;

/* Bytes of the state arena for `cfg`. Depends on the shapes only, never on a prefix
 * length (the views are fixed-size: Figure 1 caption, abstract). 0 if cfg is invalid. */
LS_API size_t ls_state_bytes(const ls_config* cfg);

/* Fills *out with the arena layout for `cfg` (host-only computation). */
LS_API int ls_get_layout(const ls_config* cfg, ls_layout* out);

/* Validates cfg, records d_arena (>= ls_state_bytes(cfg) bytes, 256-byte aligned,
 * caller-owned), zeroes it on `stream` (len = 0, every view empty) and creates the
 * host handle in *out. The arena must stay allocated until ls_destroy_state.        */
LS_API int ls_init_state(const ls_config* cfg, void* d_arena, size_t arena_bytes, ls_state** out,
                  cudaStream_t stream);

/* Workspace bytes that ls_prefill_summary needs for rows [row_begin, row_end). */
LS_API size_t ls_prefill_workspace_bytes(const ls_config* cfg, int64_t row_begin, int64_t row_end);

/* Summary initialisation over the prefix at target prefill (Figure 3 caption).
 * Appends prefix rows p in [row_begin, min(row_end, prefix_len[b])) of every sequence.
 *   d_k, d_v       element (b, l, p, h, d) at d_k[(b*L + l)*plane_stride
 *                  + (p - row_begin)*row_stride + h*D + d]  (`dtype`); row_stride >= Hkv*D,
 *                  both strides multiples of 8 elements, pointers 16-byte aligned.
 *   d_prefix_len   int64 [b]: final prefix length P_b of each sequence (0 <= P_b).
 *   row_begin/end  chunk of positions. Chunks must be passed in order starting at 0,
 *                  row_begin a multiple of the largest scale, on a state that holds
 *                  exactly min(row_begin, P_b) rows of each sequence. One call with
 *                  [0, max P_b) prefills everything.
 *   d_last_hidden  [b][L][hidden] hidden vectors at position P_b - 1 (becomes the
 *                  boundary view) or NULL to leave the boundary untouched.
 *   d_workspace    >= ls_prefill_workspace_bytes(...) bytes of caller scratch.
 * After the call len = min(row_end, P_b), the window holds the last min(len, W) rows,
 * the summary covers rows [0, len).                                                  */
LS_API int ls_prefill_summary(ls_state* st, const void* d_k, const void* d_v, int64_t plane_stride,
                       int64_t row_stride, const int64_t* d_prefix_len, int64_t row_begin,
                       int64_t row_end, const void* d_last_hidden, void* d_workspace,
                       size_t workspace_bytes, cudaStream_t stream);

/* Prefill that allocates nothing (the paper has no counterpart: this is an interface
 * for callers that cannot allocate device memory when they prefill, e.g. an inference
 * engine that reserves nearly all of the GPU's memory for its own KV-cache pool at
 * start-up, so a cudaMalloc would fail or break up that pool, or a C host that links
 * only this library and has no device allocator of its own).
 * Same arguments and result as ls_prefill_summary, without the workspace: the unit sums
 * live in a fixed array of 16 MiB compiled into the library; every GPU that loads the
 * library holds it until the process exits. Each call needs
 * ls_prefill_workspace_bytes(cfg, row_begin, row_end) <= 16 MiB, otherwise it returns
 * LS_ERR_SCRATCH_LIMIT and does nothing: split the prefix into chunks (row_begin a
 * multiple of the largest scale) that each fit. The first call for a state's device
 * looks up that device's copy of the array (cudaGetSymbolAddress, with the state's
 * device current); make that first call before any stream capture. Every call uses the same array, which keeps the last call's contents (nothing
 * in it has to start at zero), so calls that overlap on the GPU race: order them on one
 * stream or with events. Calls no cudaMalloc/cudaFree and no allocating routine.      */
LS_API int ls_prefill_summary_noalloc(ls_state* st, const void* d_k, const void* d_v,
                                      int64_t plane_stride, int64_t row_stride,
                                      const int64_t* d_prefix_len, int64_t row_begin,
                                      int64_t row_end, const void* d_last_hidden,
                                      cudaStream_t stream);

/* One round's view extraction from the target's verification pass (Figure 2 (a)-(b),
 * Figure 3 caption). Verify row 0 is the previous round's bonus token, rows 1..B the
 * B drafts; target_ids[i] is the target's greedy choice after verify row i.
 *   d_draft_ids     int32 [b][B];   d_target_ids int32 [b][B+1]
 *   d_verify_k/v    `dtype` [b][L][B+1][Hkv][D]
 *   d_verify_hidden `dtype` [b][L][B+1][hidden]
 *   d_accept_len    int32 [b] out: a;  d_next_token int32 [b] out: target_ids[a]
 * Retains verify rows 0..a (Delta = a + 1 <= B + 1): ring window, summary sums,
 * segment finalisation and mean rows, boundary = verify_hidden[a], len += Delta.   */
LS_API int ls_commit_round(ls_state* st, const int32_t* d_draft_ids, const int32_t* d_target_ids,
                    const void* d_verify_k, const void* d_verify_v,
                    const void* d_verify_hidden, int32_t* d_accept_len,
                    int32_t* d_next_token, cudaStream_t stream);

/* Stochastic acceptance for sampled decoding (T > 0; Table 1 against the greedy Table 3).
 * The pages print no rule for it; this is standard speculative sampling (Leviathan,
 * Kalman and Matias 2023; Chen et al. 2023), made position by position over the block:
 *   d_draft_ids    int32 [b][B]          the block's draft tokens
 *   d_draft_probs  fp32  [b][B][vocab]    the drafter's distribution q_i at block position i
 *   d_target_probs fp32  [b][B+1][vocab]  the target's distribution p_i after verify row i
 *   d_uniforms     fp32  [b][B+1]        draws in [0, 1): u_0..u_{B-1} for the tests, u_B for
 *                                        the final draw
 *   d_accept_len   int32 [b] out: a = the number of leading drafts kept, draft i kept iff
 *                  u_i * q_i(d_i) < p_i(d_i) (fp32 product and comparison)
 *   d_next_token   int32 [b] out: drawn from max(0, p_a - q_a) when a < B, from p_B when
 *                  a = B: the first token t whose running sum over tokens 0..t exceeds
 *                  u_B times the total (fp32 sums in the kernel's order). A residual
 *                  with no mass (p_a <= q_a everywhere) is replaced by p_a itself, so
 *                  the token is always one the target gives mass.
 * vocab a multiple of 4 and <= 524288 (else LS_ERR_SHAPE / LS_ERR_UNSUPPORTED); the
 * probability pointers 16-byte aligned. Reads 2B gathered values per sequence and the
 * draw's row(s) once (plus the drawn 8192-entry chunk again). A draft id outside
 * [0, vocab), or a target row drawn from with no mass (next token 0), sets
 * LS_DEVERR_SAMPLE. The state only lends its
 * shapes and a scratch region (sequences may not run two of these calls at once). Feed
 * the accepted counts to ls_commit_accepted.                                          */
LS_API int ls_accept_sampled(ls_state* st, const int32_t* d_draft_ids, const float* d_draft_probs,
                             const float* d_target_probs, int32_t vocab, const float* d_uniforms,
                             int32_t* d_accept_len, int32_t* d_next_token, cudaStream_t stream);

/* The drafter's projections ahead of its attention: boundary keys/values from the
 * boundary view and block queries from the drafter's block inputs (Figure 2 caption (c):
 * the drafter uses the views; the pages do not describe its learned projections, so this
 * is a plain linear map per tapped layer, no bias, fp32 accumulation):
 *   d_w_kv  bf16 [L][2 Hkv D][hidden]  rows g D + d: key of KV head g; Hkv D + g D + d: value
 *   d_w_q   bf16 [L][Hq D][hidden]     rows qh D + d: query head qh
 *   d_x     bf16 [b][L][B][hidden]     the drafter's block inputs
 *   d_bkv   bf16 [b][L][2 Hkv D] out   bkv[b][l][n] = sum_k W_kv[l][n][k] boundary[b][l][k]
 *   d_q     bf16 [b][L][B][Hq D] out   q[b][l][i][n] = sum_k W_q[l][n][k] x[b][l][i][k]
 * The boundary hidden vectors are the state's boundary view. The outputs feed
 * ls_draft_attend: d_q as its queries, boundary_k = d_bkv, boundary_v = d_bkv + Hkv D,
 * boundary_stride = 2 Hkv D. Runs on the tcgen05 tensor cores: needs a bf16 state,
 * hidden a multiple of 64, Hq D and 2 Hkv D multiples of 128 (else LS_ERR_UNSUPPORTED);
 * pointers 16-byte aligned. Boundary tiles left over after whole waves of CTAs are split
 * along the hidden size; their fp32 partial sums use the state's prologue scratch
 * (ls_layout.off_prologue), so two calls on one state must not overlap on the GPU (order
 * them on one stream). Repeated calls give the same bits. The kernel is launched as the
 * programmatic dependent of the kernel before it on `stream` and streams the weights
 * before that kernel has completed (the block inputs and the boundary view only after):
 * d_w_kv and d_w_q, the drafter's parameters, must not be written by the kernel launched
 * just before this call on the stream.                                                  */
LS_API int ls_draft_prologue(const ls_state* st, const void* d_w_kv, const void* d_w_q, const void* d_x,
                             void* d_bkv, void* d_q, cudaStream_t stream);

/* ls_commit_round with the accepted counts given (d_accept_len int32 [b], e.g. from
 * ls_accept_sampled) instead of the greedy scan; the next tokens are the caller's. A
 * count outside [0, B] sets LS_DEVERR_SAMPLE and is clamped. Other arguments as
 * ls_commit_round.                                                                     */
LS_API int ls_commit_accepted(ls_state* st, const int32_t* d_accept_len, const void* d_verify_k,
                              const void* d_verify_v, const void* d_verify_hidden, cudaStream_t stream);

/* The drafter's block attention over the three views (Figure 2 (c)).
 *   layers [layer_begin, layer_begin + layer_count)
 *   d_q            `dtype` [b][layer_count][B][Hq][D]
 *   d_out          same shape; fp32 with LS_FLAG_OUT_F32, else `dtype`
 *   d_boundary_k/v `dtype`, element (b, l, g, d) at [(b*L + l)*boundary_stride + g*D + d]
 *                  with l the absolute layer; boundary_stride >= Hkv*D, multiple of 8.
 *   softmax_scale  logit multiplier, finite and > 0 (1/sqrt(D) for the usual attention).
 * Uses the tcgen05 tensor-core kernel when dtype is bf16, (Hq/Hkv)*B == 64, D == 128 and
 * kv_rows <= 768 (unless LS_FLAG_FORCE_SIMT), otherwise a CUDA-core kernel. The
 * tensor-core kernel is launched as the programmatic dependent of the kernel before it
 * on `stream`: it reads the inputs that kernel may write only once that kernel has
 * completed. When no commit or prefill has written this state's views since another call
 * on the state was launched on the same stream (per-layer calls, or the call after
 * ls_draft_prologue), it loads its first rows of the views before that, so its start
 * overlaps the end of the kernel before it. Inside a stream capture it does not (the
 * order of the graph's replays is not known when it is captured), and a call captured
 * into a graph counts as no such earlier call for the calls launched directly after the
 * capture (they follow whatever was launched on the stream before it). A caller that writes
 * the arena itself (a checkpoint restored into it) does so with a copy, or a kernel that
 * does not trigger programmatic dependents before it completes (any kernel launched
 * without that trigger, as a plain copy kernel is).                                     */
LS_API int ls_draft_attend(const ls_state* st, int32_t layer_begin, int32_t layer_count,
                    const void* d_q, const void* d_boundary_k, const void* d_boundary_v,
                    int64_t boundary_stride, float softmax_scale, void* d_out,
                    cudaStream_t stream);

/* ls_draft_attend over a subset of the views: the drafter of a component ablation
 * (Table 5: without the global summary, without the boundary state, without the recent
 * KV window). `views` is a non-zero OR of LS_VIEW_*; the rows of the other views take
 * no part in the softmax, and the kernels do not read them where whole 128-row chunks
 * (or the summary rows of the last chunk) belong to left-out views. A query row whose
 * remaining views hold no valid row (e.g. the window alone before the first commit)
 * gets an all-zero output. `views` may also hold LS_ATTEND_INPUTS_READY. Other
 * arguments and errors as ls_draft_attend; LS_ERR_INVALID_ARG when `views` names no
 * view or has bits outside LS_VIEW_ALL | LS_ATTEND_INPUTS_READY.                    */
LS_API int ls_draft_attend_views(const ls_state* st, int32_t layer_begin, int32_t layer_count,
                                 const void* d_q, const void* d_boundary_k, const void* d_boundary_v,
                                 int64_t boundary_stride, float softmax_scale, int32_t views,
                                 void* d_out, cudaStream_t stream);

/* Bytes of the drafting state that a drafter with the given views keeps (the state-size
 * side of Table 5): the counters always; LS_VIEW_WINDOW the ring rows (b*L*Hkv*W*2*D
 * elements); LS_VIEW_SUMMARY the fp32 segment means, partial and global sums plus their
 * attention-dtype copies (b*L*Hkv*2*D*(nsc*(slots+1)+1) of each); LS_VIEW_BOUNDARY the
 * boundary hidden vectors (b*L*hidden elements). Region sizes without the 256-byte
 * alignment padding that ls_state_bytes adds between regions. 0 for an invalid config
 * or `views` outside LS_VIEW_ALL.                                                   */
LS_API size_t ls_view_state_bytes(const ls_config* cfg, int32_t views);

/* ---- the same calls reading the target's paged KV cache (no dense staging) -------
 * Prefill: ls_prefill_summary with the prefix rows of sequence b at positions
 * 0 .. P_b - 1 read from `kv` (h_kv: host pointer to the descriptor, read during the call
 * only). d_workspace may be NULL: the unit sums then live in the library's fixed 16 MiB
 * array (the rules of ls_prefill_summary_noalloc apply, LS_ERR_SCRATCH_LIMIT included).
 * Positions past max_blocks * page_size, or pages outside [0, num_pages), set
 * LS_DEVERR_PAGE.                                                                     */
LS_API int ls_prefill_paged(ls_state* st, const ls_paged_kv* h_kv, const int64_t* d_prefix_len,
                            int64_t row_begin, int64_t row_end, const void* d_last_hidden, void* d_workspace,
                            size_t workspace_bytes, cudaStream_t stream);

/* ls_commit_round with verify row i's keys/values read from `kv` at the target's position
 * len_b + i (len_b: the rows the state holds; the verify pass wrote rows 0..B there).
 * Only the retained rows 0..a are read. The hidden vectors stay a dense input.        */
LS_API int ls_commit_round_paged(ls_state* st, const int32_t* d_draft_ids, const int32_t* d_target_ids,
                                 const ls_paged_kv* h_kv, const void* d_verify_hidden, int32_t* d_accept_len,
                                 int32_t* d_next_token, cudaStream_t stream);

/* ls_commit_accepted (given counts) reading the verify rows from `kv` as above.        */
LS_API int ls_commit_accepted_paged(ls_state* st, const int32_t* d_accept_len, const ls_paged_kv* h_kv,
                                    const void* d_verify_hidden, cudaStream_t stream);

/* ls_round with the commit reading `kv` (ls_commit_round_paged, then the attention).    */
LS_API int ls_round_paged(ls_state* st, const int32_t* d_draft_ids, const int32_t* d_target_ids,
                          const ls_paged_kv* h_kv, const void* d_verify_hidden, int32_t* d_accept_len,
                          int32_t* d_next_token, const void* d_q, int64_t boundary_k_offset,
                          int64_t boundary_v_offset, float softmax_scale, void* d_out, cudaStream_t stream);

/* One whole decoding round: ls_commit_round, then ls_draft_attend over all layers, for
 * drafters whose boundary keys/values are slices of the new boundary hidden vector:
 * element (b, l, g, d) of the boundary key is hidden_b,l[boundary_k_offset + g*D + d] and
 * of the value hidden_b,l[boundary_v_offset + g*D + d], hidden_b,l being verify row a's
 * hidden vector (offsets multiples of 8, each slice inside `hidden`). Arguments as in the
 * two calls; the result (state, accept_len, next_token, out) is the same as theirs.
 * Where the tcgen05 kernel applies (ls_round_overlaps) the attention kernel is launched
 * as a programmatic dependent of the commit kernel: it is scheduled while the commit runs,
 * sets itself up and loads its first Q tile, then waits on the device for the commit's
 * writes. d_q must therefore be complete when the call is issued (stream order gives
 * that), and must not be written by the commit's outputs.                              */
LS_API int ls_round(ls_state* st, const int32_t* d_draft_ids, const int32_t* d_target_ids,
                    const void* d_verify_k, const void* d_verify_v, const void* d_verify_hidden,
                    int32_t* d_accept_len, int32_t* d_next_token, const void* d_q,
                    int64_t boundary_k_offset, int64_t boundary_v_offset, float softmax_scale,
                    void* d_out, cudaStream_t stream);

/* 1 if ls_round overlaps the attention kernel's launch with the commit for this state
 * (programmatic dependent launch), 0 if it makes the two calls in turn.              */
LS_API int ls_round_overlaps(const ls_state* st);

/* 1 if ls_draft_attend takes the tcgen05 path for this state, 0 if the CUDA-core one. */
LS_API int ls_attend_uses_tensor_cores(const ls_state* st);

/* Copies the first `bytes` bytes of the arena to h_dst; synchronises `stream`. */
LS_API int ls_read_state(const ls_state* st, void* h_dst, size_t bytes, cudaStream_t stream);

/* Reads the device error word into *h_code (synchronous). Returns LS_ERR_DEVICE or
 * LS_ERR_DEVICE_TIMEOUT when it is non-zero, LS_OK otherwise.                      */
LS_API int ls_get_error(const ls_state* st, int32_t* h_code);

/* Clears the device error word (enqueued on `stream`). The word is sticky otherwise: a
 * bit once set stays until this call or a fresh ls_init_state. Also zeroes the arrival
 * counts that a call which gave up part-way (LS_DEVERR_WAIT_TIMEOUT) may have left in the
 * arena (commit, ls_accept_sampled, ls_draft_prologue), so that later calls count right;
 * the views themselves are whatever that call left (restore a checkpoint if needed).    */
LS_API int ls_clear_error(ls_state* st, cudaStream_t stream);

/* Check of the device-side failure detection: one kernel polls an mbarrier that nothing
 * signals, gives up after `polls` polls (1 .. 2^22; each poll suspends for at most a
 * hardware-chosen interval), sets LS_DEVERR_WAIT_TIMEOUT in the error word and returns,
 * as every bounded wait of the path kernels does when a partner never arrives. The next
 * ls_get_error reports LS_ERR_DEVICE_TIMEOUT; the context stays usable (ls_clear_error,
 * then carry on).                                                                      */
LS_API int ls_check_wait_timeout(ls_state* st, uint32_t polls, cudaStream_t stream);

/* Frees the host handle only; the arena stays the caller's. */
LS_API void ls_destroy_state(ls_state* st);

/* Static description of a status code. */
LS_API const char* ls_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* LONGSPARK_H_ */
