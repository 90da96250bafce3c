/*
 * ep.h — C ABI of the B200 (sm_100a) MoE expert-parallel dispatch / combine
 * library, libep_b200.so.
 *
 * What the operations are (the pages describe them in words, without
 * formulas; citations are page title + section):
 *  - dispatch sends every token to the k experts its router picked and
 *    returns the received tokens, their gate weights and a handle; combine
 *    brings the experts' outputs back to each token's rank and sums them
 *    using that handle; the same handle serves combine_backward and
 *    dispatch_backward ("DeepEP：MoE 专家并行 EP 通信 kernel 编译与使用指南"
 *    (zhouruolin.cn), section 五 使用方法 and FAQ Q5).
 *  - FP8 dispatch with BF16 combine is the standard precision pair
 *    ("deepep-expert-parallel-communication-library" (blog.hotdry.top),
 *    section 五 实践建议; "DeepSeek 开源周第二弹" (czhn.yksolo.com): 原生 FP8
 *    调度支持), and the precision conversion is fused into the data movement
 *    ("DeepEP：专为MoE模型打造的All-to-All通信库" (bjdmk.com.cn), section 3.2).
 *  - the per-expert token counts are the quantity one inspects for load skew
 *    ("DeepEP：专为MoE模型打造的All-to-All通信库", section 5.2).
 *  - the number of SMs a call may use is a caller knob
 *    ("deepep-expert-parallel-communication-library", section 二 SM 资源控制).
 *
 * Model of the expert-parallel world: one GPU, R virtual ranks.  Rank r owns
 * source tokens [r*T/R, (r+1)*T/R) and experts [r*E/R, (r+1)*E/R).  Every
 * receive buffer is one array of rows in expert-major order; rank r's
 * partition is rows [expert_offset[r*E/R], expert_offset[(r+1)*E/R]).  Dense
 * layout: P = T*k rows, no gaps.  Padded layout (the low-latency kernels'
 * static per-expert buffers, sized by num_max_tokens_per_rank, for decoding
 * with CUDA graphs: "deepep-expert-parallel-communication-library",
 * sections 一 and 二; "DeepEP：MoE 专家并行 EP 通信 kernel 编译与使用指南",
 * section 五): E*R*M rows, see ep_shape_t.max_tokens_per_rank.
 *
 * Numerics (the pages do not fix them; these are the definitions used):
 *  - slots: the pairs routed to expert e take rows [expert_offset[e],
 *    expert_offset[e+1]) in increasing (token t, top-k position j) order,
 *    i.e. (source rank, source token) order.  topk_idx = -1 masks a pair.
 *  - FP8 (OCP E4M3, largest finite 448): per token and 128-channel group,
 *    amax = max |x| (fp32), scale = amax / 448 (fp32 IEEE division; 1.0 if
 *    that is 0), code = E4M3(x / scale) with IEEE fp32 division, round to
 *    nearest even, saturating to +-448.
 *  - combine: acc = +0.0f; acc = fmaf(w[t,j], y[slot(t,j)], acc) for
 *    j = 0..k-1 in order (masked pairs skipped); out = bf16 RNE(acc).
 *  - combine_backward: grad_y[slot(t,j)] = bf16 RNE(w[t,j] * g[t]) (one fp32
 *    product); grad_w[t,j] = sum_h g[t,h] * y[slot(t,j),h] in fp32 (the
 *    summation order is the kernel's).
 *  - dispatch_backward: grad_x[t] = bf16 RNE(sum_j grad_recv[slot(t,j)]),
 *    fp32 adds from +0.0f in j order (straight-through for FP8).
 *
 * Conventions shared by every entry point:
 *  - All array arguments are DEVICE pointers owned by the caller, except the
 *    ep_shape_t / ep_handle_t structs themselves, which are read from host
 *    memory during the call only.  The library never allocates, never frees
 *    and never synchronises the stream (except ep_get_error, and every call
 *    when the environment variable EP_DEBUG=1 is set).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Calls on one handle must not overlap; results are defined
 *    once the stream reaches them.  Below 16 tokens per SM the kernels are
 *    launched with programmatic dependent launch (EP_PDL=0 turns it off): a
 *    kernel may become resident while the previous kernel on the stream
 *    finishes, but it reads and writes no global memory before that kernel
 *    has completed, so stream order is kept for any predecessor.  (One
 *    exception inside a call: ep_dispatch_with_layout's dispatch reads x while
 *    the call's own layout still runs, which never writes x; everything
 *    before the call has completed by then.)
 *  - The one-launch layout (up to 16384 pairs) runs as one thread-block
 *    cluster of 16 CTAs, a non-portable cluster size, where the device can
 *    hold one, else 8; EP_LAYOUT_CLUSTER=8 keeps it at 8.
 *  - bf16 arrays are uint16 bit patterns; rows of bf16 / fp8 arrays must start
 *    on 16-byte boundaries (H % 8 == 0 and 16-byte aligned base pointers).
 *  - Return value: EP_OK or an ep_status_t code.  Argument errors are found
 *    on the host before anything is enqueued.  Out-of-range expert ids are
 *    found on the device: the pair is treated as masked and bit 0 of
 *    handle->error_word is set; ep_get_error reports it.
 *  - Limits: 0 <= T, T % R == 0, 1 <= k <= 32, 1 <= E <= 1024, 1 <= R <= E,
 *    R <= 256, E % R == 0, T*k < 2^31, 8 <= H, H % 8 == 0 (H % 128 == 0 with
 *    FP8), use_fp8 0 or 1, num_sms >= 0;
 *    padded layout: see max_tokens_per_rank.
 */
#ifndef EP_B200_H
#define EP_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* ep_stream_t;

typedef enum {
  EP_OK = 0,
  EP_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, shape outside the limits */
  EP_ERR_BAD_INDEX = 2,    /* a topk_idx entry outside [-1, E) (from ep_get_error) */
  EP_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed */
  EP_ERR_UNSUPPORTED = 4,  /* the current device is not an sm_100 GPU */
  EP_ERR_SCRATCH_TOO_SMALL = 5, /* the shape needs more layout scratch than
                                   ep_get_dispatch_layout_noalloc's fixed array */
  EP_ERR_CAPACITY = 6           /* padded layout: some (source rank, expert) block got more
                                   than max_tokens_per_rank pairs (from ep_get_error) */
} ep_status_t;

/* Problem shape. T tokens over R virtual ranks, hidden H, top-k, E experts. */
typedef struct {
  int32_t T, H, k, E, R;
  int32_t use_fp8; /* 1: dispatch writes E4M3 codes + fp32 scales; 0: bf16 rows */
  int32_t num_sms; /* SM budget of the data-movement kernels (dispatch,
                      combine, both backward passes) and the router: 0 or a
                      value >= the device's SM count = all SMs; else each of
                      their grids is capped at num_sms x (CTAs of that kernel
                      resident per SM), so the caller's own kernels keep the
                      rest ("deepep-expert-parallel-communication-library",
                      section 二 SM 资源控制).  The hardware places a grid's
                      CTAs on distinct SMs before it stacks them, so the CTAs
                      land on num_sms SMs only when the stream belongs to an
                      SM partition of that size (a CUDA green context).  The
                      layout kernels (microseconds; the one-launch layout is
                      one cluster of 16 or 8 CTAs) are not capped.  Results
                      do not depend on the budget. */
  int32_t max_tokens_per_rank; /* 0: dense receive layout (below).  M > 0:
                      the padded low-latency layout: E*R*M receive rows, one
                      block of M rows per (expert e, source rank r) at row
                      (e*R + r)*M; the pair (t, j) takes row (e*R + r)*M + i,
                      i its position among rank r's pairs to e in (t, j)
                      order.  Needs M >= T/R, E*R*M < 2^31, (T/R)*k <= 8192.
                      Pairs past M get no row (EP_ERR_CAPACITY via
                      ep_get_error; only duplicate experts in a row can cause
                      it).  Rows with no pair are not written. */
} ep_shape_t;

/* The dispatch handle: device arrays written by ep_get_dispatch_layout and
 * read by the other calls.  Sizes are given by ep_handle_sizes. */
typedef struct {
  int32_t* num_tokens_per_expert;  /* [E]   pairs routed to each expert */
  int32_t* expert_offset;          /* [E+1] exclusive prefix sum of the above */
  int32_t* num_tokens_per_rank;    /* [R]   tokens with >= 1 pair on rank r */
  int32_t* count_src_rank_expert;  /* [R*E] pairs from source rank r to expert e (padded: may exceed M) */
  int32_t* src_rank_expert_offset; /* [R*E] first row of (source rank r, expert e) */
  uint8_t* is_token_in_rank;       /* [T*R] 1 if token t has a pair on rank r */
  int32_t* slot_of_pair;           /* [T*k] receive row of pair (t,j); -1 if masked */
  int32_t* src_of_slot;            /* [rows] t*k+j of the pair in each receive row, -1 if none;
                                      rows = T*k (dense) or E*R*M (padded) */
  int32_t* error_word;             /* [1]   device error bits; must be 0 before first use */
} ep_handle_t;

/* Element counts of each handle array, in struct order (9 entries). */
int ep_handle_sizes(const ep_shape_t* shape, int64_t counts[9]);

/* Bytes of device scratch ep_get_dispatch_layout needs (a multiple of 256). */
size_t ep_workspace_size(const ep_shape_t* shape);

/* Routing layout: per-expert and per-rank histograms, offsets,
 * is_token_in_rank and the slot of every (token, expert) pair.
 * topk_idx: [T,k] int64 row-major, device.  workspace: device scratch of at
 * least ep_workspace_size bytes, 256-byte aligned, contents irrelevant.
 * Three kernels: tile histograms, column scans, slot assignment. */
int ep_get_dispatch_layout(const ep_shape_t* shape, const int64_t* topk_idx,
                           const ep_handle_t* handle, void* workspace,
                           size_t workspace_bytes, ep_stream_t stream);

/* Dispatch: x [T,H] bf16 -> recv_x [P,H] (bf16, or E4M3 codes when
 * use_fp8), recv_scale [P,H/128] fp32 (required with use_fp8, else ignored),
 * recv_weight [P] fp32 = topk_weights of each row's pair (may be NULL).
 * topk_weights [T,k] fp32.  Rows past expert_offset[E] are not written. */
int ep_dispatch(const ep_shape_t* shape, const void* x, const float* topk_weights,
                const ep_handle_t* handle, void* recv_x, float* recv_scale,
                float* recv_weight, ep_stream_t stream);

/* Layout and dispatch in one call, as the pages' dispatch takes x and
 * topk_idx together and returns the received tokens with the handle
 * ("DeepEP：MoE 专家并行 EP 通信 kernel 编译与使用指南" (zhouruolin.cn),
 * section 五 使用方法).  Arguments are those of ep_get_dispatch_layout and
 * ep_dispatch; every check of both runs before anything is enqueued, and the
 * results (handle, recv_x, recv_scale, recv_weight, error word) are those of
 * ep_get_dispatch_layout followed by ep_dispatch on the same stream.
 * Below 16 tokens per SM with programmatic dependent launch, when H is
 * 1536 < H <= 8192 (the bulk-store dispatch), the last layout kernel lets the
 * dispatch kernel be scheduled only after its own wait, i.e. once everything
 * enqueued before this call has completed, and each dispatch CTA then loads
 * and quantises its first x rows (one per shared-memory row stage) while
 * the layout still runs, sending them once their slots are known (the
 * layout writes only the handle and the workspace, never x). */
int ep_dispatch_with_layout(const ep_shape_t* shape, const int64_t* topk_idx, const void* x,
                            const float* topk_weights, const ep_handle_t* handle,
                            void* workspace, size_t workspace_bytes, void* recv_x,
                            float* recv_scale, float* recv_weight, ep_stream_t stream);

/* Combine: y [P,H] bf16 (expert outputs in receive order), topk_weights
 * [T,k] fp32 -> out [T,H] bf16.  A token with no valid pair gets +0. */
int ep_combine(const ep_shape_t* shape, const void* y, const float* topk_weights,
               const ep_handle_t* handle, void* out, ep_stream_t stream);

/* Backward of combine: grad_out [T,H] bf16, y [P,H] bf16, topk_weights [T,k]
 * -> grad_y [P,H] bf16 (rows of masked pairs untouched), grad_w [T,k] fp32
 * (0 for masked pairs). */
int ep_combine_backward(const ep_shape_t* shape, const void* grad_out, const void* y,
                        const float* topk_weights, const ep_handle_t* handle,
                        void* grad_y, float* grad_w, ep_stream_t stream);

/* Backward of dispatch: grad_recv [P,H] bf16 -> grad_x [T,H] bf16. */
int ep_dispatch_backward(const ep_shape_t* shape, const void* grad_recv,
                         const ep_handle_t* handle, void* grad_x, ep_stream_t stream);

/* ep_get_dispatch_layout without caller-provided scratch.  The pages describe
 * no such call (it has no counterpart there); it exists for callers that may
 * not allocate device memory: code that runs inside another framework's
 * allocator or memory-pool hooks (allocating there would re-enter that
 * allocator), and embedded or real-time hosts whose device memory is fixed
 * at start-up.  The scratch comes from one fixed array of
 * ep_noalloc_scratch_bytes() (1 MiB) inside the library, which every GPU that
 * loads the library keeps until the process exits.
 *  - Same arguments, results and argument errors as ep_get_dispatch_layout,
 *    minus the workspace.  After the shape, handle and topk_idx checks, it
 *    returns EP_ERR_SCRATCH_TOO_SMALL, and enqueues nothing, when
 *    ep_workspace_size(shape) exceeds the array (the limit is about 1000
 *    layout tiles x (E + R) columns, e.g. T = 32768, E = 256, R = 8 needs
 *    271 KiB).
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *  - The first call in each CUDA context (per device; again after
 *    cudaDeviceReset, and in each green or driver-API context) looks up the
 *    array's device address there (cudaGetSymbolAddress) and caches it for
 *    that context; make that first call before any stream capture.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; nothing in it needs to start at zero.  Calls whose kernels
 *    overlap on the GPU (other streams, other threads) race on it: order
 *    them on one stream or serialise them. */
int ep_get_dispatch_layout_noalloc(const ep_shape_t* shape, const int64_t* topk_idx,
                                   const ep_handle_t* handle, ep_stream_t stream);

/* Size in bytes of ep_get_dispatch_layout_noalloc's fixed scratch array. */
size_t ep_noalloc_scratch_bytes(void);

/* Group-limited top-k routing, the step that produces topk_idx and
 * topk_weights (experts split into groups; a token picks its best groups,
 * then its top-k experts inside them: "deepep-expert-parallel-
 * communication-library", sections 一 and 三).
 * scores: [T,E] fp32, finite, device.  Experts are n_groups groups of E /
 * n_groups consecutive ids (n_groups <= 32); a group's score is its largest
 * expert score; the topk_groups best groups are kept, then the k best
 * experts inside them, ties to the lower index.  topk_idx [T,k] int64 lists
 * them by descending score; topk_weights [T,k] fp32 = softmax of their
 * scores.  Needs k <= topk_groups * E / n_groups.  One warp per token. */
int ep_route_group_limited(const ep_shape_t* shape, const float* scores, int n_groups, int topk_groups,
                           int64_t* topk_idx, float* topk_weights, ep_stream_t stream);

/* ---- Multi-GPU expert parallelism: one process per GPU -----------------
 *
 * R ranks, one GPU each (the pages' EP8 over NVLink:
 * "deepep-expert-parallel-communication-library", section 一; dispatch and
 * combine are all-to-alls between ranks: "DeepEP：MoE 专家并行 EP 通信
 * kernel 编译与使用指南", section 五).  Rank r
 * holds tokens [r*T/R, (r+1)*T/R) and experts [r*E/R, (r+1)*E/R).  Every
 * rank gathers all ranks' topk_idx ([T,k], T*k*8 bytes) and runs
 * ep_get_dispatch_layout over it, so every rank holds the same global
 * layout.  Owner rank o keeps the global receive rows
 * [expert_offset[o*E/R], expert_offset[(o+1)*E/R]) in its own buffers, row
 * expert_offset[o*E/R] first; the concatenation over o of those buffers is
 * the single-GPU receive buffer.  The calls below move this rank's tokens
 * only, and read or write each receive row in its owner's buffer, which may
 * be another GPU's memory (a peer address reachable from this device: CUDA
 * IPC, or memory allocated for symmetric access).  Loads are plain ones;
 * stores are plain ones or, in dispatch for 1536 < H <= 8192, TMA bulk
 * copies from shared memory.  No TMA load and no multicast.  The arithmetic
 * is that of the single-GPU calls, element for element.
 *
 * shape: the global problem (T = all ranks' tokens); R <= EP_MAX_PEERS.
 * rank: this process's rank.  topk_idx: [T,k] int64, every rank's ids (the
 * layout's input).  handle: the global layout.  Per-rank arrays (x,
 * topk_weights, out, grad_out, grad_w, grad_x) hold this rank's T/R tokens.
 * Peer tables give, for every owner o < R, the base of o's buffer: rows of
 * H bf16 (or H E4M3 bytes for recv_x under FP8), H/128 fp32 scales, or one
 * fp32 weight per row; 16-byte aligned.  recv_weight may be NULL (no
 * weights written).  Same stream ordering, no allocation and no sync as the
 * single-GPU calls; the caller orders the ranks' calls (a barrier or
 * events between a buffer's writers and its readers). */
#define EP_MAX_PEERS 64
typedef struct {
  void* rows[EP_MAX_PEERS];
} ep_peer_rows_t;

int ep_dispatch_peers(const ep_shape_t* shape, int32_t rank, const int64_t* topk_idx, const ep_handle_t* handle,
                      const void* x, const float* topk_weights, const ep_peer_rows_t* recv_x,
                      const ep_peer_rows_t* recv_scale, const ep_peer_rows_t* recv_weight, ep_stream_t stream);
int ep_combine_peers(const ep_shape_t* shape, int32_t rank, const int64_t* topk_idx, const ep_handle_t* handle,
                     const ep_peer_rows_t* y, const float* topk_weights, void* out, ep_stream_t stream);
int ep_combine_backward_peers(const ep_shape_t* shape, int32_t rank, const int64_t* topk_idx,
                              const ep_handle_t* handle, const void* grad_out, const ep_peer_rows_t* y,
                              const float* topk_weights, const ep_peer_rows_t* grad_y, float* grad_w,
                              ep_stream_t stream);
int ep_dispatch_backward_peers(const ep_shape_t* shape, int32_t rank, const int64_t* topk_idx,
                               const ep_handle_t* handle, const ep_peer_rows_t* grad_recv, void* grad_x,
                               ep_stream_t stream);

/* Peer buffers between processes (one process per GPU, or several on one
 * GPU): how a rank obtains the addresses of the other ranks' buffers for the
 * peer tables above, through CUDA IPC.  The EP world is built from a process
 * group ("DeepEP：MoE 专家并行 EP 通信 kernel 编译与使用指南", section 五
 * 使用方法), and inside one node the ranks reach each other's memory directly
 * ("deepep-expert-parallel-communication-library", section 四).  Host calls
 * only: nothing is enqueued and nothing is allocated.
 *
 * ep_ipc_export: describes the device buffer at `ptr` (any address inside a
 * cudaMalloc allocation of the calling process, e.g. a tensor of torch's
 * default caching allocator; not stream-ordered pool or virtual-memory
 * allocations, which give EP_ERR_CUDA) as a plain 80-byte record that can be
 * sent to the other processes (handle of the whole allocation, the buffer's
 * offset in it, and the bytes from there to the allocation's end).  The
 * exporting process keeps the allocation alive, and does not free or reuse
 * it, until every importer has closed its mapping.
 * ep_ipc_open: maps another process's exported buffer into this process (on
 * this process's current device; the exporter's GPU may be another one with
 * peer access, or the same one) and returns the mapping's base, to be given
 * to ep_ipc_close, and the buffer's address in it, for the peer tables.  A
 * process must not open its own export.  Opening the same allocation again
 * returns the same mapping; each open needs its own close.
 * ep_ipc_close: unmaps one open (its mapped_base), after the last kernel that
 * reads or writes through it has finished.
 *
 * Ordering between ranks (a buffer's writers before its readers) stays the
 * caller's: for example, every rank synchronises its stream and then meets
 * the others at a host barrier between dispatch and combine. */
typedef struct {
  unsigned char handle[64]; /* cudaIpcMemHandle_t of the allocation */
  uint64_t offset;          /* the buffer's byte offset inside the allocation */
  uint64_t bytes;           /* bytes from the buffer's start to the allocation's end */
} ep_ipc_buffer_t;

int ep_ipc_export(const void* ptr, ep_ipc_buffer_t* out);
int ep_ipc_open(const ep_ipc_buffer_t* buf, void** mapped_base, void** ptr);
int ep_ipc_close(void* mapped_base);

/* Synchronises `stream`, reads handle->error_word, clears it, and returns
 * EP_ERR_BAD_INDEX if a bad expert id was seen since the last read, else
 * EP_ERR_CAPACITY if a padded block overflowed, else EP_OK; EP_ERR_CUDA if
 * the stream reports an error. */
int ep_get_error(const ep_handle_t* handle, ep_stream_t stream);

/* Static description of a status code. */
const char* ep_status_string(int status);

/* Text of the last CUDA error seen by this thread ("" if none). */
const char* ep_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* EP_B200_H */
