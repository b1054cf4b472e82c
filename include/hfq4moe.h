/*
 * hfq4moe.h - C ABI of libhfq4moe.so: the routed-expert MoE layer of LLM
 * decode over HFQ4 block-quantised expert weights, on NVIDIA B200 (sm_100a).
 *
 * Sources (page title and section):
 *   [HFQ]   hipfire RDNA engine forum thread, section "HFQ quantisation format
 *           and GEMV optimisation": 256-weight blocks of 136 bytes, an f32
 *           scale, an f32 zero point and 128 bytes of packed 4-bit data;
 *           decode is a bandwidth-bound GEMV over such blocks.
 *   [TOPK]  hipfire MoE expert-offload explainer, opening section: each token
 *           activates 8 of its layer's experts (top-8 routing).
 *   [PLACE] same explainer, section "placement algorithm": layer split
 *           VRAM_LAYERS=N, auto fit-capacity placement, expert hot set, loud
 *           refusal naming the byte deficit.
 *   [PCIE]  same explainer, section "PCIe pass-through": host-mapped pinned
 *           expert weights are read by the GPU kernel directly over PCIe,
 *           with no staging copy.
 *   [TABLE] Strata user report, section "model and engine": a per-(layer,
 *           expert) offset table locates every expert's gate/up/down bytes.
 *   [ARENA] Strata user report, pitfall 7: the pinned expert arena is
 *           registered with the CUDA runtime, 2 MiB pages when available.
 *   [WMMA]  gfx1151 engine README, Windows section: a self-written matrix-
 *           core GEMM for prefill (prior art for the tensor-core path).
 *   [CACHE] Strata user report, section "model and engine": hot experts in a
 *           VRAM cache in front of the pinned host arena.
 *
 * Conventions shared by every entry point:
 *   - Weights: w = zero + scale * q with q in [0, 15].  Block layout: f32
 *     scale, f32 zero (little-endian), 128 bytes of nibbles, byte j holding
 *     element 2j in its low nibble and 2j+1 in its high nibble.  A matrix of
 *     R rows x C columns is R x ceil(C/256) blocks, row after row; a row
 *     shorter than a whole number of blocks is padded with q = 0.
 *   - A packed expert is [gate I x H][up I x H][down H x I] matrices, back
 *     to back (hfq4_expert_bytes(H, I) bytes).  At H = 2048, I = 512 that is
 *     1,671,168 bytes, a multiple of 256.
 *   - Ownership: the caller allocates and owns every buffer (device memory
 *     normally comes from the caller's allocator).  The library allocates
 *     only the pinned host arenas that hfq_host_arena_create makes, and
 *     never allocates on the forward path: scratch is the caller's
 *     workspace, sized by the *_workspace_bytes queries.
 *   - Streams: `stream` is a cudaStream_t passed as void*; NULL means the
 *     legacy default stream.  GPU work is asynchronous on it.
 *   - Errors: every call returns an hfq_status; argument errors are found on
 *     the host before anything is launched and leave outputs untouched.
 *     hfq_last_error() returns a thread-local message for the last failure.
 *     Device-side conditions (a bounded wait that ran out) are written to a
 *     status word in the workspace and read by hfq_workspace_status().
 *   - Limits: 1 <= k <= 16, k <= E <= 512, H and I multiples of 128
 *     (H, I <= 8192), T <= 65536, pointers 16-byte aligned.
 */
#ifndef HFQ4MOE_H
#define HFQ4MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HFQ_OK = 0,
    HFQ_ERR_ARG = -1,          /* a size, count or pointer argument is invalid */
    HFQ_ERR_ALIGN = -2,        /* a pointer is not 16-byte aligned */
    HFQ_ERR_UNSUPPORTED = -3,  /* a shape outside the limits above */
    HFQ_ERR_NOFIT = -4,        /* placement does not fit the HBM budget */
    HFQ_ERR_CUDA = -5,         /* a CUDA runtime call failed */
    HFQ_ERR_TIMEOUT = -6,      /* a bounded device-side wait ran out */
    HFQ_ERR_ALLOC = -7,        /* host arena allocation or registration failed */
    HFQ_ERR_WORKSPACE = -8     /* workspace missing or smaller than required */
} hfq_status;

typedef enum { HFQ_F32 = 0, HFQ_BF16 = 1 } hfq_dtype;

/* Which expert path hfq4_moe_forward runs. */
typedef enum {
    HFQ_PATH_AUTO = 0,  /* GEMV when tokens per expert are few, else tensor cores */
    HFQ_PATH_GEMV = 1,  /* CUDA-core HFQ4 GEMV (decode, speculative verify) */
    HFQ_PATH_TC = 2     /* dequantise to bf16 + tcgen05 grouped GEMM (prefill) */
} hfq_path;

#define HFQ4_BLOCK 256
#define HFQ4_BLOCK_BYTES 136
#define HFQ_MAX_EXPERTS 512
#define HFQ_MAX_TOPK 16
#define HFQ_MAX_STACK_LAYERS 64

/* Message of the last failed call on this thread ("" if none). */
const char *hfq_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int hfq_version(void);

/* Bytes of an HFQ4 matrix [HFQ]: rows * ceil(cols / 256) * 136.  0 on bad args. */
size_t hfq4_matrix_bytes(int rows, int cols);

/* Bytes of one packed expert: 2 * matrix(I, H) + matrix(H, I).  0 on bad args. */
size_t hfq4_expert_bytes(int hidden, int inter);

/*
 * Quantise and pack experts on the host [HFQ].
 *   gate, up: f32 [n_experts][inter][hidden], row-major, host memory.
 *   down:     f32 [n_experts][hidden][inter].
 *   out:      host buffer of at least n_experts * hfq4_expert_bytes(hidden,
 *             inter) bytes; expert e starts at e * hfq4_expert_bytes.
 * Per block (the real elements of a row only): scale = f32(f32(max - min) /
 * 15), zero = min, q = clamp(rint(f32(f32(w - zero) / scale)), 0, 15),
 * rounding half to even; scale == 0 stores q = 0.  Inputs must be finite.
 * Single-threaded, deterministic, bit-identical to the device variant.
 */
hfq_status hfq4_pack_experts(const float *gate, const float *up, const float *down,
                             int n_experts, int hidden, int inter, void *out, size_t out_bytes);

/* Same as hfq4_pack_experts with device pointers, asynchronous on `stream`. */
hfq_status hfq4_pack_experts_device(const float *gate, const float *up, const float *down,
                                    int n_experts, int hidden, int inter, void *out,
                                    size_t out_bytes, void *stream);

/*
 * Dequantise one HFQ4 matrix (device) [HFQ]: out[r][c] = fmaf(scale, q, zero),
 * the correctly rounded f32 of zero + scale*q, for r < rows, c < cols.
 *   blocks: device, hfq4_matrix_bytes(rows, cols) bytes, 8-byte aligned.
 *   out:    device f32 [rows][cols].
 */
hfq_status hfq4_dequant(const void *blocks, int rows, int cols, float *out, void *stream);

/*
 * Top-k softmax routing with renormalised weights [TOPK] (device).
 *   logits: f32 [T][E].
 *   idx:    int32 [T][k] out: the k experts with the largest logits, slot 0
 *           the largest; equal logits go to the lower expert index.
 *   wts:    f32 [T][k] out: p_j / sum_selected p, p = softmax(logits); this
 *           is the softmax over the selected logits.
 *   cnt, off, perm: optional grouping by expert (all three or none):
 *           cnt int32 [E] pairs per expert, off int32 [E+1] exclusive prefix
 *           sum, perm int32 [T*k] the pair ids t*k+j of expert e at
 *           perm[off[e] .. off[e+1]), ascending.
 *   workspace: needed only with grouping, hfq_route_workspace_bytes(T, E, k)
 *           bytes of device scratch (may be NULL when that is 0).
 * NaN logits are not supported.
 */
size_t hfq_route_workspace_bytes(int T, int E, int k);
hfq_status moe_route(const float *logits, int T, int E, int k, int32_t *idx, float *wts,
                     int32_t *cnt, int32_t *off, int32_t *perm, void *workspace,
                     size_t ws_bytes, void *stream);

/*
 * Router logits (device): logits[t][e] = sum_c x[t][c] * Wr[e][c], the plain
 * linear map of each token's hidden state that picks its layer's experts
 * (hipfire offload explainer, opening section: each token's router selects 8
 * of the layer's experts; no bias).
 *   x:      [T][hidden] in x_dtype (f32 or bf16), 16-byte aligned.
 *   router: Wr [n_experts][hidden] in router_dtype (f32 or bf16), 16-byte
 *           aligned.  hidden must be a multiple of 8.
 *   logits: f32 [T][n_experts] out.
 * Summation order (fixed, so every call and the fused router in the decode
 * stack give the same bits): 256 partial sums p_j, j = 32*g + lane
 * (g = 0..7), each taking the 8-column chunks c0 = 8*j + 2048*i in turn (the
 * chunk's products in order, fused multiply-add); each group g's 32 partials
 * added by a butterfly over the lanes (xor 16, 8, 4, 2, 1); the group sums
 * added as ((q0+q1)+(q2+q3))+((q4+q5)+(q6+q7)).  Returns HFQ_ERR_ARG /
 * HFQ_ERR_ALIGN on bad arguments, HFQ_ERR_UNSUPPORTED beyond the limits,
 * HFQ_ERR_CUDA on a launch error.
 */
hfq_status moe_router_logits(const void *x, hfq_dtype x_dtype, int T, int hidden, const void *router,
                             hfq_dtype router_dtype, int n_experts, float *logits, void *stream);

/*
 * One MoE layer's experts [TABLE][PCIE].
 *   expert_ptr: DEVICE array [n_experts] of base addresses of the packed
 *               experts, each 16-byte aligned; an address may be HBM or a
 *               host-mapped pinned buffer (see hfq_host_arena_create).
 *   expert_loc: DEVICE array [n_experts] (or NULL = all HBM): 0 = HBM,
 *               1 = host-mapped.  Host-mapped experts are read over PCIe by
 *               the same kernel, with plain loads.
 */
typedef struct {
    const void *const *expert_ptr;
    const uint8_t *expert_loc;
    int n_experts;
    int hidden;
    int inter;
} hfq4_layer;

/*
 * Routed experts of one layer for T tokens (device):
 *   y[t] = sum_j wts[t][j] * Wd_e (silu(Wg_e x_t) * (Wu_e x_t)),  e = idx[t][j],
 * summed in slot order j with fp32 accumulation.
 *   x:      [T][H] in x_dtype (f32 or bf16).
 *   idx, wts: routing as written by moe_route ([T][k]).
 *   cnt, off, perm: grouping by expert (from moe_route); required for
 *           HFQ_PATH_TC; with AUTO and T > 8 they select the tensor-core
 *           path, without them T > 8 runs the per-layer GEMV kernels.
 *   path:   AUTO: T <= 8 -> persistent GEMV kernel; T > 8 with grouping ->
 *           tensor cores where the shape allows them (hidden and inter
 *           multiples of 128, each with an even number of 256-weight blocks
 *           per row, so that rows are whole 16-byte units for the tensor
 *           maps), else the per-layer GEMV kernels.  GEMV forces CUDA cores;
 *           TC forces the tensor-core path (HFQ_ERR_UNSUPPORTED for other
 *           shapes) [WMMA]: weights dequantised to RN_bf16(fmaf(scale, q, zero)),
 *           x rounded to bf16 (exact for bf16 input), f32 accumulation, h
 *           carried into the down projection as two bf16 parts (hi and the
 *           bf16 rounding of h - hi, about 16 significant bits), each pair's down
 *           output kept in f32 and y summed over the k slots in slot order
 *           (deterministic).
 *   y:      f32 [T][H] out.  y_bf16: optional bf16 [T][H] out (NULL = none).
 *   workspace: hfq4_moe_workspace_bytes(T, k, H, I, E) bytes of device
 *           scratch (plus the same again for HFQ_PATH_TC with T <= 8),
 *           256-byte aligned, zero-filled before first use, owned by the
 *           caller; calls that share a workspace must be ordered on one stream.
 */
size_t hfq4_moe_workspace_bytes(int T, int k, int hidden, int inter, int n_experts);
hfq_status hfq4_moe_forward(const hfq4_layer *layer, const void *x, hfq_dtype x_dtype, int T,
                            const int32_t *idx, const float *wts, int k, const int32_t *cnt,
                            const int32_t *off, const int32_t *perm, float *y, void *y_bf16,
                            int path, void *workspace, size_t ws_bytes, void *stream);

/*
 * A decode stack of MoE layers joined by a bf16 residual stream (device):
 * for l = 0 .. n_layers-1, route layer l on logits[l] (top-k softmax,
 * renormalised), run its experts on x_l, then x_{l+1} = bf16(x_l + y_l).
 * Layer l's logits are read only after layer l-1 has finished, as a router
 * that depends on x_l would require.  One kernel per layer, or one
 * persistent kernel for the whole stack (HFQ_PATH_AUTO/GEMV).
 *   layers:  host array [n_layers] of layer descriptors (n_layers <= 64),
 *            all with the same n_experts, hidden, inter.
 *   logits:  f32 [n_layers][T][E] (device).
 *   x0:      bf16 [T][H] (device), the residual stream entering layer 0.
 *   x_out:   bf16 [T][H] out, the residual after the last layer (may alias
 *            nothing else).
 *   y_all:   optional f32 [n_layers][T][H] out: every layer's y (NULL = none).
 *   idx_all, wts_all: optional int32/f32 [n_layers][T][k] out (NULL = none).
 *   T <= 8.  workspace: hfq4_stack_workspace_bytes(T, k, H, I, E) bytes.
 */
size_t hfq4_stack_workspace_bytes(int T, int k, int hidden, int inter, int n_experts);
/* Kernel launches one hfq4_moe_decode_stack call makes (1 when the whole stack
 * runs as one persistent launch, 3 per layer otherwise); 0 on bad arguments. */
int hfq4_stack_launches(int n_layers, int T, int k, int hidden, int inter);
hfq_status hfq4_moe_decode_stack(const hfq4_layer *layers, int n_layers, const float *logits,
                                 int k, const void *x0, int T, void *x_out, float *y_all,
                                 int32_t *idx_all, float *wts_all, int path, void *workspace,
                                 size_t ws_bytes, void *stream);

/*
 * The same decode stack with each layer's router in the loop: layer l's
 * logits are computed from x_l by moe_router_logits' arithmetic (same bits)
 * instead of being read from memory, so the residual stream decides the
 * routing as in the model.
 *   router:  Wr [n_layers][E][H] in router_dtype (f32 or bf16, device,
 *            16-byte aligned).
 *   logits_all: optional f32 [n_layers][T][E] out: every layer's logits.
 *   The other arguments as for hfq4_moe_decode_stack (path AUTO).  With
 *   T = 1, a bf16 router and a shape the persistent kernel takes, the whole
 *   stack, routers included, is one launch: every CTA computes a share of
 *   the logits and the shares are exchanged through the workspace.
 *   Otherwise each layer is a router launch followed by a one-layer stack.
 *   workspace: hfq4_stack_workspace_bytes(T, k, H, I, E) bytes.
 */
hfq_status hfq4_moe_decode_stack_routed(const hfq4_layer *layers, int n_layers, const void *router,
                                        hfq_dtype router_dtype, int k, const void *x0, int T,
                                        void *x_out, float *y_all, int32_t *idx_all, float *wts_all,
                                        float *logits_all, void *workspace, size_t ws_bytes,
                                        void *stream);

/*
 * Allocation-free variant of hfq4_moe_forward.  The pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory or
 * hand the library a workspace - for example code that runs while a framework
 * is capturing a stream into a CUDA graph with its own allocator, serving
 * loops that forbid any allocation after start-up, or plugins whose host
 * application gives them no allocator.  It computes the same y as
 * hfq4_moe_forward (same kernel, same arguments minus the workspace and path)
 * and allocates nothing: its scratch is one fixed array of device memory
 * inside the library (548 KiB; every GPU that loads the library holds it until
 * the process exits).
 *   Limits: 1 <= T <= 8, k <= 16, inter <= 1024, hidden <= 2048; anything
 *   larger returns HFQ_ERR_UNSUPPORTED naming the limit.
 *   The first call on a device looks up the array's device address for that
 *   device (with that device current).  Each call clears the array's control
 *   words on `stream` before
 *   launching, the status word among them.  All calls share the one array, so
 *   calls that overlap on the GPU (different streams without ordering) race;
 *   order them on one stream.  Calls may change k, T and the layer's shape
 *   from one to the next: a one-token call whose exchange layout (k, inter,
 *   hidden) differs from the last one's clears the array's h part first.
 *   Device-side conditions (a bounded wait that ran out, an expert id outside
 *   [0, n_experts)) go to the array's status word: read it with
 *   hfq_workspace_status(NULL, 0, stream) after the call and before the next
 *   one, which clears it.
 */
hfq_status hfq4_moe_forward_noalloc(const hfq4_layer *layer, const void *x, hfq_dtype x_dtype,
                                    int T, const int32_t *idx, const float *wts, int k, float *y,
                                    void *y_bf16, void *stream);

/*
 * Library options (process-wide, host side):
 *   HFQ_OPT_WAIT_TIMEOUT_NS: deadline of every bounded device-side wait
 *     (grid barriers, expert counters, ring barriers), default 1 s.  When a
 *     wait runs out, the kernel records HFQ_ERR_TIMEOUT in the workspace
 *     status word, stops doing work, lets its copies in flight land and exits.
 *   HFQ_OPT_TEST_MISSING_ARRIVALS: fault injection for tests; the next
 *     persistent-kernel launch makes its grid barriers wait for this many
 *     CTAs that do not exist (the one-token kernel, which has no grid
 *     barrier: makes its layer-1 input poll, or with one layer its h poll,
 *     expect a tag nobody writes), so the wait runs out without any fault.
 *   HFQ_OPT_TIMELINE_BUFFER: debug; the device address of a u64 buffer of
 *     n_sms * n_layers * 32 words, zero-filled (0 = off).  Persistent-kernel
 *     launches then write %globaltimer stamps (ns), per layer l at word
 *     (row * n_layers + l) * 32 + s.  The one-token and general kernels write
 *     rows 0 and 1 (CTA 0 and CTA gridDim/2): [0] layer start, [1] routed,
 *     [2] table built, [3 + s] ring stage s ready (s < 12), [16] gate/up done,
 *     [17] all h ready, [18] h staged, [19] down done, [20] layer end, [21]
 *     all copies issued, [22 + s] bytes of stage s landed (s < 10).  The
 *     2..8-token kernel writes row c for every CTA c: [0] layer start, [1]
 *     inputs and routing done, [2] pair table built, [3] first gate/up item
 *     landed, [4] gate/up done, [5] h exchange done, [6] down done, [7]
 *     outputs written, [8] last gate/up item issued, [9] all items issued.
 * Returns HFQ_ERR_ARG for an unknown option or a value out of range.
 */
#define HFQ_OPT_WAIT_TIMEOUT_NS 1
#define HFQ_OPT_TEST_MISSING_ARRIVALS 2
#define HFQ_OPT_TIMELINE_BUFFER 3
hfq_status hfq_set_option(int option, long long value);

/*
 * Device status word of a workspace (synchronises `stream`): HFQ_OK,
 * HFQ_ERR_TIMEOUT if a bounded device-side wait of a previous call ran out, or
 * HFQ_ERR_ARG if a kernel met an expert id outside [0, n_experts) or (tensor-
 * core path) a grouping whose cnt/off/perm do not describe the T*k pairs; the
 * work of such a pair is skipped, its output left unwritten.  After an error
 * the word and the workspace's control block are cleared.  A new workspace
 * must be zero-filled before its first use.  workspace = NULL with
 * ws_bytes = 0 reads the status word of hfq4_moe_forward_noalloc's array on
 * the current device (HFQ_OK when no such call has run there).
 */
hfq_status hfq_workspace_status(void *workspace, size_t ws_bytes, void *stream);

/*
 * Pinned, mapped host arena for offloaded experts [PCIE][ARENA].
 *   bytes:   arena size.
 *   flags:   HFQ_ARENA_HUGEPAGE asks for 2 MiB transparent huge pages
 *            (madvise) before registration; it silently falls back to 4 KiB.
 *   host:    out, host address of the arena.
 *   dev:     out, the device address of the same memory (for expert_ptr).
 * Returns HFQ_ERR_ALLOC with the byte count in the message when pinning fails.
 * The library owns the arena until hfq_host_arena_destroy(host).
 */
#define HFQ_ARENA_HUGEPAGE 1
hfq_status hfq_host_arena_create(size_t bytes, int flags, void **host, void **dev);
hfq_status hfq_host_arena_destroy(void *host);

/*
 * Expert placement [PLACE] (host only, no allocation).
 *   counts:   uint32 [L][E] calibration selection counts (decode heat).
 *   resident_layers: N >= 0 keeps layers 0..N-1 fully in HBM; -1 = auto:
 *            the largest N for which N full layers plus the hot sets of the
 *            other L-N layers fit hbm_budget.
 *   hot_per_layer: h >= 0; in every host layer its h most selected experts
 *            (ties to the lower index) are placed in HBM too.
 *   loc_out:  uint8 [L][E] out: 0 = HBM, 1 = host.
 *   slot_out: int64 [L][E] out: index of the expert within its location's
 *            arena, numbered in (layer, expert) order.
 *   hbm_needed, host_needed: out, bytes per location.
 * Returns HFQ_ERR_NOFIT, with the deficit in the message and both byte
 * counts filled in, when the HBM part exceeds hbm_budget (loud refusal).
 */
hfq_status hfq_placement_build(int L, int E, size_t expert_bytes, const uint32_t *counts,
                               int resident_layers, int hot_per_layer, size_t hbm_budget,
                               uint8_t *loc_out, int64_t *slot_out, size_t *hbm_needed,
                               size_t *host_needed);

/*
 * Pointer table from a placement (host only): out[l*E + e] = base + slot *
 * expert_bytes with base = hbm_base for loc 0 and host_dev_base for loc 1.
 */
hfq_status hfq_placement_pointers(int L, int E, size_t expert_bytes, const uint8_t *loc,
                                  const int64_t *slot, const void *hbm_base,
                                  const void *host_dev_base, uint64_t *out);

/*
 * Expert cache over host-mapped experts [CACHE][PCIE] (host; copies and table
 * writes asynchronous on `stream`).
 *
 * Keeps up to `slots` experts of each layer in HBM slots (`slot_mem`, caller
 * device memory of L * slots * expert_bytes bytes) and maintains the layers'
 * pointer tables `table_dev` (caller device memory [L][E] u64: the
 * expert_ptr the kernels read) and, if given, location tables `loc_dev`
 * ([L][E] u8: the expert_loc they read): an entry names the expert's slot
 * while it is cached (location 0) and its home otherwise.  home, host_src and
 * home_loc are host arrays [L][E]: the address the kernels read when the
 * expert is not cached (HBM, or the device alias of a host-mapped expert),
 * its pinned host address when it lives in host memory (copy source; 0 for
 * experts resident in HBM, which are never cached), and 1 for host experts.
 * table_dev = NULL keeps the bookkeeping only (no device work; policy tests).
 * The library allocates a small host object, a pinned staging buffer of
 * 18 L E bytes, 3 L events and one stream for refill copies;
 * hfq_cache_destroy waits for its copies and frees them.
 *
 * hfq_cache_observe: the n expert ids (host array, [0, E)) one step selected
 * in `layer`.  Each distinct selected expert counts as a hit when the kernels
 * read it from HBM (resident or cached) and as a miss otherwise; its selection
 * frequency grows by one (all of the layer's frequencies are halved every 256
 * observations of the layer).  Missed experts are then admitted, most
 * frequent first (ties to the lower id), up to max_admit of them: into a free
 * slot, or in place of the least frequent cached expert not selected in this
 * call when the newcomer is more frequent.  max_admit = -1 admits every
 * missed expert whatever the frequencies (copy-engine staging before use, as
 * long as the slots hold them).  The call waits only for the table copies
 * of its layer's previous call (they read the layer's staging buffers), not
 * for the rest of `stream`.  Then it enqueues on `stream` the layer's tables
 * with evicted experts back home.  With max_admit = -1 it then enqueues on
 * `stream` the copies of the admitted experts from pinned host memory into
 * their slots (cudaMemcpyAsync: the copy engine) and the tables naming those
 * slots, so the next kernel reads them from HBM.  With max_admit >= 0
 * (refill) the copies run on the cache's own stream, behind every kernel
 * enqueued on `stream` so far (they may still read the victims' slots), and
 * overlap the kernels enqueued next.  Their slots are named at the start of
 * the layer's next call, or by hfq_cache_flush, behind those copies; until
 * then the kernels read those experts from their homes and
 * hfq_cache_slot_of reports -1 for them.  Kernels enqueued on `stream`
 * before a call may still run and read the old tables and slot contents, so
 * a step's routing can be observed while the next step runs.  No kernel that
 * reads these tables may run on another stream.
 * [CACHE] Strata report, "model and engine": a VRAM cache of hot experts in
 * front of the pinned host arena, refilled from it.
 */
typedef struct hfq_cache hfq_cache;
hfq_status hfq_cache_create(int L, int E, size_t expert_bytes, int slots, const uint64_t *home,
                            const uint64_t *host_src, const uint8_t *home_loc, void *slot_mem,
                            size_t slot_bytes, uint64_t *table_dev, uint8_t *loc_dev, void *stream,
                            hfq_cache **out);
hfq_status hfq_cache_observe(hfq_cache *cache, int layer, const int32_t *ids, int n, int max_admit,
                             void *stream);
/* Names the slots of every layer's refills in flight (see hfq_cache_observe),
 * enqueued on `stream` behind their copies. */
hfq_status hfq_cache_flush(hfq_cache *cache, void *stream);
/* Slot of an expert (-1: not cached, or its refill not yet named). */
hfq_status hfq_cache_slot_of(const hfq_cache *cache, int layer, int expert, int *slot);
/* Counters since creation (any pointer may be NULL). */
hfq_status hfq_cache_stats(const hfq_cache *cache, uint64_t *hits, uint64_t *misses,
                           uint64_t *admitted, uint64_t *evicted);
hfq_status hfq_cache_destroy(hfq_cache *cache);

/*
 * Read-bandwidth probe: a streaming kernel that reads `bytes` from `src`
 * (HBM or host-mapped) `iters` times with 16-byte loads and writes one
 * checksum word to `sink` (device).  Time it with events on `stream`.
 */
hfq_status hfq_probe_read(const void *src, size_t bytes, int iters, uint64_t *sink, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HFQ4MOE_H */
