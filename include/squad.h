/*
 * squad.h - C ABI of libsquad, SQuad-Attention on NVIDIA B200 (sm_100a).
 *
 * The operator is the two-pass attention of "SQuad: Sub-Quadratic Attention
 * Distillation for Efficient Video Generation" (gist.science technical
 * summary, Methodology section 1, "SQuad-Attention Operator"; complexity claim
 * O(n sqrt n) in the abstract):
 *
 *   tokens of a T x H x W latent grid, flattened p = (t*H + y)*W + x;
 *   local pass  (per window of tT x tH x tW tokens, w = tT*tH*tW):
 *       O1 = softmax(s * Q_w K_w^T) V_w
 *   global pass (per group of the m = n/w tokens that share the same
 *       in-window position (t mod tT, y mod tH, x mod tW)):
 *       O  = softmax(s * Q_g K_g^T) O1_g
 *   with the same input Q and K in both passes and s = 1/sqrt(d) unless the
 *   caller gives another scale. The result is O (no residual, no mask).
 *
 * Conventions shared by every entry point:
 *   - Tensors are dense, row-major [B, heads, n, d] with n = T*H*W (token
 *     order as above); LSE vectors are [B, heads, n] float32, natural log.
 *   - dtype SQUAD_BF16: q, k, v, o, o1, dout, dq, dk, dv are bfloat16 and the
 *     kernels accumulate in fp32 (tcgen05 tensor cores). SQUAD_F32: all of
 *     them are float32 and the kernels run fp32 FMA on the CUDA cores.
 *   - Every pointer is a DEVICE pointer on the current CUDA device and must
 *     be 16-byte aligned. The caller owns all memory; the library never
 *     allocates, frees or synchronises in these calls. All work is enqueued
 *     on `stream` (a cudaStream_t; NULL is the legacy default stream).
 *   - Arguments are checked before anything is launched; on any error
 *     nothing is enqueued. No entry point throws across the ABI.
 */
#ifndef SQUAD_H_
#define SQUAD_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQUAD_OK = 0,
  SQUAD_ERR_INVALID_ARG = 1,  /* NULL descriptor or required pointer, unknown dtype */
  SQUAD_ERR_SHAPE = 2,        /* non-positive size, tile does not divide grid, size overflow */
  SQUAD_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned */
  SQUAD_ERR_UNSUPPORTED = 4,  /* valid operator, but outside what the kernels handle (see below) */
  SQUAD_ERR_CUDA = 5,         /* a CUDA runtime or driver call failed (see squad_last_cuda_error) */
  SQUAD_ERR_TIMEOUT = 6,      /* a kernel gave up on a bounded wait (see squad_poll_device_error) */
  SQUAD_ERR_WORKSPACE = 7,    /* workspace missing or smaller than squad_attn_workspace_size */
  SQUAD_ERR_INDEX = 8         /* a shuffle kernel met a row index out of range (squad_poll_device_error) */
} squad_status;

typedef enum { SQUAD_F32 = 0, SQUAD_BF16 = 1 } squad_dtype;

typedef struct {
  int B, heads, d;  /* batch, heads, head dimension */
  int T, H, W;      /* latent grid; n = T*H*W */
  int tT, tH, tW;   /* window tile; must divide T, H, W */
  int dtype;        /* squad_dtype */
  float scale;      /* softmax scale; <= 0 selects 1/sqrt(d) */
} squad_desc;

/* Limits of the kernels (SQUAD_ERR_UNSUPPORTED beyond them):
 *   bf16: d in {64, 128}; tW <= 128 and W/tW <= 128 (a window row or a
 *         group row must fit one 128-token tile); B*heads*n < 2^31.
 *   f32:  d a multiple of 32, d <= 256; B*heads*n < 2^31.
 * Any w and m are accepted otherwise (the bf16 kernels tile a window or a
 * group into boxes of at most 128 tokens and run an online softmax across
 * them). */

/* Bytes of device workspace the call needs.
 *   which = 0: squad_attn_fwd with o1 == NULL: the local-pass output plus
 *              B*heads progress counters (rounded up to 256 bytes each part).
 *   which = 2: squad_attn_fwd with o1 != NULL: the counters only. With less
 *              than this (e.g. no workspace) the forward still runs, as two
 *              separate launches instead of one fused launch.
 *   which = 1: squad_attn_bwd (dO1 in the input dtype, the global-pass parts
 *              of dQ and dK in fp32, and two fp32 row vectors).
 * Returns SQUAD_OK and writes *bytes, or an argument/shape error. */
squad_status squad_attn_workspace_size(const squad_desc* desc, int which, size_t* bytes);

/* Forward: o = SQuad-Attention(q, k, v).
 *   With enough workspace (see squad_attn_workspace_size) the bf16 path runs
 *   as one launch in which the global pass of each (batch, head) starts as
 *   soon as that head's local pass is done, while its Q, K and O1 are still in
 *   L2; the counters in the workspace order the two. When o1 is NULL, the
 *   local-pass rows are also dropped from L2 after their single use. When the
 *   Q, K and O1 rows of three (batch, head) slices (3 * 3 * n * d elements)
 *   exceed 60% of the device's L2, the two passes run as two launches
 *   instead, with the same results: the global pass would read them from DRAM
 *   either way, and two launches then take less time.
 *   o1   : [B,heads,n,d] local-pass output, written when non-NULL (needed by
 *          the backward); when NULL the workspace holds it.
 *   lse1 : [B,heads,n] local-pass log-sum-exp, written when non-NULL.
 *   lse2 : [B,heads,n] global-pass log-sum-exp, written when non-NULL.
 *   workspace / workspace_bytes: see squad_attn_workspace_size(desc, 0, ..).
 * Inputs must not alias outputs. */
squad_status squad_attn_fwd(const squad_desc* desc, const void* q, const void* k, const void* v, void* o,
                            void* o1, float* lse1, float* lse2, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Forward from host memory. q, k, v and o are HOST pointers ([B, heads, n, d]
 * of the descriptor's dtype; pinned memory for the copies to overlap, pageable
 * memory works but serialises). The (batch, head) slices are independent, so
 * the call runs on chunks of slices_per_chunk slices: the copy of chunk i+1 to
 * the device (on stream_in), the forward of chunk i (on stream, as
 * squad_attn_fwd without o1) and the copy of chunk i-1 back (on stream_out)
 * overlap. Results are those of squad_attn_fwd, bitwise. The call is ordered
 * after the work already on `stream`, and o is complete once `stream` has been
 * synchronised (all three streams join it). The three streams must differ.
 * workspace: device, 16-byte aligned, at least
 * squad_attn_fwd_host_workspace_size bytes (two sets of chunk buffers and the
 * chunk forward's workspace), owned by the caller, not shared with a call in
 * flight. Events are created and released inside the call. */
squad_status squad_attn_fwd_host_workspace_size(const squad_desc* desc, int slices_per_chunk, size_t* bytes);
squad_status squad_attn_fwd_host(const squad_desc* desc, const void* q, const void* k, const void* v, void* o,
                                 int slices_per_chunk, void* workspace, size_t workspace_bytes,
                                 void* stream, void* stream_in, void* stream_out);

/* One pass of the forward, for callers that compose or time the passes on
 * their own. stage 1 (local pass): out = per-window attention with values
 * `val` = v. stage 2 (global pass): out = per-group attention with values
 * `val` = the stage-1 output. lse (may be NULL) receives that pass's
 * log-sum-exp. squad_attn_fwd is stage 1 followed by stage 2 on one stream. */
squad_status squad_attn_fwd_pass(const squad_desc* desc, int stage, const void* q, const void* k,
                                 const void* val, void* out, float* lse, void* stream);

/* Forward that allocates nothing, not even a workspace. The paper has no
 * counterpart: this entry point exists for callers that cannot hand the
 * library device memory for scratch, e.g. code running inside a host
 * framework that owns every device allocation (a fixed memory pool or arena)
 * and forbids side allocations, or latency-critical code that must not call
 * cudaMalloc because it may synchronise the device. Such callers pass only
 * their inputs and outputs; the local-pass output, which squad_attn_fwd keeps
 * in o1 or in the caller's workspace, lives here in a fixed 32 MiB array of
 * device memory inside the library (SQUAD_NOALLOC_SCRATCH_BYTES).
 *   - Limit: B*heads*n*d*sizeof(element) must fit in that array (bf16: at most
 *     16,777,216 elements, fp32: 8,388,608); larger problems are rejected
 *     with SQUAD_ERR_WORKSPACE before anything is launched.
 *   - Every GPU that loads the library holds the array until the process
 *     exits. The first call on a device looks up the array's device address
 *     (a cudaGetSymbolAddress with that device current) and caches it; make
 *     that first call before any stream capture.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents. Each call overwrites every element it later reads, so nothing
 *     needs clearing, but calls whose kernels overlap on the GPU (different
 *     streams, or different host threads) race on the array: serialise them.
 *   - Arguments are those of squad_attn_fwd with o1 == NULL; lse1 and lse2 may
 *     be NULL. The two passes run as two launches (squad_attn_fwd fuses them
 *     into one); each row is computed by the same kernel code, and the results
 *     agree with squad_attn_fwd's within the tolerances its tests state. */
#define SQUAD_NOALLOC_SCRATCH_BYTES (32u << 20)
squad_status squad_attn_fwd_noalloc(const squad_desc* desc, const void* q, const void* k, const void* v,
                                    void* o, float* lse1, float* lse2, void* stream);

/* Backward of the forward for the loss sum(o * dout): writes dq, dk, dv.
 * o, o1, lse1, lse2 are the forward's outputs for the same q, k, v (all
 * required). The global pass is differentiated first (values o1), then the
 * local pass (values v); dq and dk sum both passes' contributions.
 * bf16: when a window or group spans several 128-row boxes, the parts of dq
 * from its key boxes are added in fp32 with atomic reductions in whatever
 * order the hardware runs them, so dq may differ between runs in the last
 * fp32 bits before its final bf16 rounding; dk, dv and the forward are
 * bitwise reproducible. */
squad_status squad_attn_bwd(const squad_desc* desc, const void* q, const void* k, const void* v,
                            const void* o, const void* o1, const float* lse1, const float* lse2,
                            const void* dout, void* dq, void* dk, void* dv, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ---- More than two passes ----
 * The pages name composing more than two passes as an outlook ("SQuad:
 * Sub-Quadratic Attention Distillation for Efficient Video Generation",
 * gist.science technical summary, Significance and Claims). Reading: k =
 * ntiles + 1 passes over nested tiles t_1 | t_2 | ... | t_{k-1} | grid, given
 * as tiles[3*ntiles] = (tT, tH, tW) innermost first, each dividing the next
 * (and the last the grid) along every axis; desc->tT, tH, tW are ignored and
 * 1 <= ntiles <= 4. Pass j attends among the tokens that share a t_j-window and
 * the position inside their t_{j-1}-window (t_0 = one token, t_k = the grid);
 * its values are the output of pass j-1 (v for j = 1); q, k and the scale are
 * those of every pass; the result is the output of pass k. ntiles = 1 is
 * the operator of squad_attn_fwd with tile t_1. Cost: 4 n d (|t_1| +
 * |t_2|/|t_1| + ... + n/|t_{k-1}|) FLOPs per (batch, head). On bf16 with a
 * workspace the k passes run in one launch, pass j of a (batch, head) starting
 * once pass j-1 of it is done (the results are bitwise those of one launch per
 * pass); otherwise each pass is one launch. On bf16 the
 * forward packs the problems of a pass several to a tensor-core box when they
 * have at most 64 tokens and the problem box has an extent-1 dimension (a
 * per-row key mask keeps them apart); the results then equal the unpacked
 * ones up to fp32 summation order. On bf16 every pass's box row (t_j / t_{j-1}
 * along W) must be at most 128 tokens (else SQUAD_ERR_UNSUPPORTED); tiles
 * that do not nest give SQUAD_ERR_SHAPE. */

/* Bytes of workspace squad_attn_multi_fwd needs. save_inter != 0 (the caller
 * passes inter): one uint32 counter per (pass 2..k, batch, head), for the
 * one-launch bf16 forward. save_inter == 0 (inter NULL): first the k-1
 * intermediate outputs, then the counters. Each part is 256-byte aligned. */
squad_status squad_attn_multi_fwd_workspace_size(const squad_desc* desc, int ntiles, const int* tiles,
                                                 int save_inter, size_t* bytes);

/* Forward. inter: ntiles consecutive [B, heads, n, d] tensors of the input
 * dtype receiving the outputs of passes 1..k-1 (each is the next pass's values,
 * and the backward reads them), or NULL for inference: they then live in the
 * workspace, and on bf16 each row leaves L2 without being written back once
 * the next pass has read it (when its problem fits one box). lse: k
 * consecutive [B, heads, n] fp32 (natural log), or NULL. workspace: device,
 * 16-byte aligned, at least squad_attn_multi_fwd_workspace_size bytes for the
 * same save_inter (else SQUAD_ERR_WORKSPACE), owned by the caller and
 * overwritten, not read; NULL (allowed only with inter) runs one launch per
 * pass; it must not be shared with a call in flight on another stream. On f32
 * only its intermediate part is used. o, inter, lse (and the workspace) are
 * written, nothing else. */
squad_status squad_attn_multi_fwd(const squad_desc* desc, int ntiles, const int* tiles, const void* q,
                                  const void* k, const void* v, void* o, void* inter, float* lse, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Bytes of workspace squad_attn_multi_bwd needs: two upstream-gradient
 * tensors of the input dtype, four fp32 [B, heads, n, d] accumulators and
 * three fp32 row vectors (each part 256-byte aligned). */
squad_status squad_attn_multi_bwd_workspace_size(const squad_desc* desc, int ntiles, const int* tiles,
                                                 size_t* bytes);

/* Backward for the loss sum(o * dout): writes dq, dk, dv. o, inter and lse
 * (all required) are squad_attn_multi_fwd's outputs for the same inputs. The
 * passes are differentiated from the last to the first; dq and dk sum every
 * pass's contribution (in fp32 until the last step). The bf16 dq is
 * reproducible only up to the fp32 reduction order when a problem spans
 * several boxes (as for squad_attn_bwd). */
squad_status squad_attn_multi_bwd(const squad_desc* desc, int ntiles, const int* tiles, const void* q,
                                  const void* k, const void* v, const void* o, const void* inter, const float* lse,
                                  const void* dout, void* dq, void* dk, void* dv, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* ---- Sequence-parallel forward over G ranks ----
 * Sharded by windows, the local pass needs nothing from other ranks, and the
 * global pass needs one row of every window for each in-window position (the
 * operator of "SQuad: Sub-Quadratic Attention Distillation for Efficient Video
 * Generation", gist.science technical summary, Methodology section 1). Rank r
 * holds the tokens of a contiguous range of whole tT-frame windows (frames
 * split as evenly as the frame windows allow) and, for the global pass, a range
 * of in-window positions (split as evenly as possible). The forward on each rank:
 *   1. local pass on its shard (squad_attn_fwd_pass, stage 1, grid T_r x H x W);
 *   2. squad_sp_pack of Q, K and the local-pass output with map send1;
 *   3. all-to-all (the caller's collective, e.g. NCCL) with counts send1/recv1;
 *   4. squad_sp_unpack with maps recv1_src/recv1_row into the position-major
 *      layout [position][window], which is the grid (P_r*T/tT) x (H/tH) x (W/tW)
 *      with tile (T/tT) x (H/tH) x (W/tW): each of its windows is one global-pass
 *      group, so
 *   5. the global pass is squad_attn_fwd_pass stage 1 on that grid;
 *   6. squad_sp_pack of its output with map send2, all-to-all with counts
 *      send2/recv2, squad_sp_unpack with recv2_src/recv2_row: the output rows
 *      back in the shard's token order.
 * No counterpart in the pages beyond the operator itself; the exchange is the
 * plainest one the two passes allow. desc describes the whole problem; G ranks
 * (1..64, at most the number of frame windows and of positions). */

/* info[8]: [0] first frame of rank `rank`, [1] its frames, [2] its tokens n_local
 * (= frames*H*W), [3] its position-major rows n_pos (= positions*m), [4] its
 * first position, [5] its positions, [6] w, [7] m. Host only. */
squad_status squad_sp_plan_info(const squad_desc* desc, int G, int rank, int* info);

/* The index maps of rank `rank` (host arrays, in rows of one (batch, head) slice):
 * counts[4*G] = rows per peer of send1, recv1, send2, recv2 (in that order);
 * send1[n_local], recv1_src[n_pos], recv1_row[n_pos], send2[n_pos],
 * recv2_src[n_local], recv2_row[n_local] (meaning as in the steps above). Host only. */
squad_status squad_sp_plan_maps(const squad_desc* desc, int G, int rank, int* counts, int* send1, int* recv1_src,
                                int* recv1_row, int* send2, int* recv2_src, int* recv2_row);

/* Pack rows for an all-to-all: dst holds, peer after peer, [tensor][slice][counts[q]]
 * rows; row i of peer q, tensor t, slice s is row idx[prefix_q + i] of slice s of
 * srcs[t] (srcs: ntensors <= 3 device tensors [slices, rows_in, row_bytes]).
 * counts: host [G]; idx: device int32 [sum counts]; row_bytes a multiple of 16.
 * An index outside [0, rows_in) skips that row and sets the device error word. */
squad_status squad_sp_pack(const void* const* srcs, int ntensors, int slices, int rows_in, int row_bytes, int G,
                           const int* counts, const int* idx, void* dst, void* stream);

/* Unpack rows received from an all-to-all (src laid out as squad_sp_pack writes, with
 * counts[q] rows per slice from peer q): row j of slice s of dsts[t] is row src_row[j]
 * of peer src_rank[j]'s block for tensor t, slice s. dsts: ntensors device tensors
 * [slices, rows_out, row_bytes]; src_rank, src_row: device int32 [rows_out]. An out
 * of range peer or row skips that row and sets the device error word. */
squad_status squad_sp_unpack(const void* src, int ntensors, int slices, int rows_out, int row_bytes, int G,
                             const int* counts, const int* src_rank, const int* src_row, void* const* dsts,
                             void* stream);

/* Geometry the kernels use for one pass (stage 1 = local/window pass,
 * stage 2 = global/cross-window pass), for tests and byte accounting.
 * Writes 8 ints to info: [0] rows per problem (w or m), [1] problems per
 * (batch, head), [2] tensor-core tiles per problem, [3] rows per tile box,
 * [4] box extent along a, [5] along b, [6] along c, [7] key tiles held per
 * online-softmax group. No CUDA call is made. */
squad_status squad_plan_info(const squad_desc* desc, int stage, int* info);

/* Self-test of the device timeout path (no counterpart in the paper): launches
 * one small kernel whose thread waits, through the same bounded wait the
 * attention kernels use, on a barrier that nothing ever completes. After
 * timeout_ns (1 us .. 10 s) it gives up and sets the device error word, so a
 * following squad_poll_device_error returns SQUAD_ERR_TIMEOUT and clears it.
 * Nothing faults or hangs and the context stays usable. */
squad_status squad_selftest_wait_timeout(unsigned long long timeout_ns, void* stream);

/* Synchronises `stream`, then reads and clears the library's device error
 * word. Returns SQUAD_ERR_TIMEOUT if a kernel gave up on a bounded wait since
 * the last poll, SQUAD_ERR_INDEX if a shuffle kernel skipped a row whose index
 * was out of range, SQUAD_ERR_CUDA if the synchronisation failed, else SQUAD_OK. */
squad_status squad_poll_device_error(void* stream);

/* Human-readable name of a status code (static storage). */
const char* squad_strerror(int status);

/* cudaError_t / CUresult value of the last failing CUDA call on this thread. */
int squad_last_cuda_error(void);

/* Counters of the library's tensor-map cache (no counterpart in the paper). Every
 * call that launches a tensor-core kernel needs TMA tensor maps (eight per forward
 * launch, four per backward pass); their encoding is a host driver call, and maps
 * already made for the same device, pointers and shapes are reused instead: hits
 * counts the reused ones, misses the encoded ones, since the library was loaded and
 * over all threads. Either pointer may be NULL (not both). No CUDA call is made. */
squad_status squad_tmap_cache_stats(unsigned long long* hits, unsigned long long* misses);

/* Library version: major * 10000 + minor * 100 + patch. */
int squad_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SQUAD_H_ */
