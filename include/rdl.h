/*
 * rdl.h -- C ABI of librdl.so: route-layer chunk-routing sparse attention on B200.
 *
 * The method is Prefilling-dLLM v2 ("Prefilling-dLLM v2: Learned Chunk Routing for
 * Long-Context Diffusion Language Models", Figure 3 caption and Table 3; explained in
 * "The 172x Speedup Has an Evidence Budget", section "How learned routing controls what
 * the model can read").  A sequence is cut into chunks of S = 64 positions: 63 content
 * tokens and one routing mask in the last slot (position 64c+63 of chunk c).
 *
 * Notation: C = L/64 chunks, G = Hq/Hkv heads per GQA group, g(h) = h / G,
 * tau = 1/sqrt(d), content(c) = {64c + j : j = 0..62}.
 * Window of a query at position p:  W(p) = { j : |p - j| <= w, 0 <= j < L }  (w < 0: empty).
 * Eligible (remote) chunks:         E(p) = { c : no position of chunk c lies in W(p) }.
 *
 * Layouts (row-major, element strides implied):
 *   q, o       [B, Lq, Hq, d]   storage dtype (bf16 or f32); a row's G heads are adjacent
 *   k, v       [B, Hkv, L, d]   storage dtype; a chunk of one KV head is one 64*d slab
 *   x          [B, Lq, D]       storage dtype;   w_down [D, r];  w_up [r, Hq*d]
 *   q_pos      [B, Lq] int32    position of each query row; NULL means row i is at
 *                               position i (then Lq must equal L)
 *   summary    [B, Hq, C, d]    fp32 (or the split layout of RDL_FLAG_SPLIT_SUMMARY);
 *                               entropy [B, Hq, C] fp32
 *   idx        [B, Hkv, Lq, K]  int32: selected chunks in ascending order, then -1
 *   z_sel      [B, Hq, Lq, K]   fp32: route score of each selected chunk for each head
 *                               (-inf in padded slots)
 *   lse        [B, Hq, Lq]      fp32, natural-log partition of each output row
 *
 * Conventions shared by every call:
 *   - All device buffers are owned by the caller.  The library never allocates, never
 *     frees and never synchronises (except rdl_last_device_status).  Work is enqueued on
 *     `stream` (a cudaStream_t passed as void*; NULL = legacy default stream).
 *   - Pointers are device pointers, 16-byte aligned; outputs must not alias inputs.
 *   - Arguments are checked on the host before any launch: an invalid value returns
 *     RDL_ERR_INVALID_ARG, a valid but unimplemented combination RDL_ERR_UNSUPPORTED,
 *     and nothing is launched.  A failed launch returns RDL_ERR_CUDA.
 *   - Kernels never trap: a device-side check that fails (debug flag RDL_FLAG_CHECKS)
 *     or a bounded wait that runs out records a code in a device status word, read
 *     back by rdl_last_device_status.
 *   - Mask-slot query rows (position % 64 == 63) are not route-layer queries: the score
 *     call writes idx = -1 / z_sel = -inf for them and rdl_route_attn leaves their o and
 *     lse rows untouched.  Their output is written by rdl_summary_pool (o_mask).
 */
#ifndef RDL_H
#define RDL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RDL_OK = 0,
  RDL_ERR_INVALID_ARG = -1,
  RDL_ERR_UNSUPPORTED = -2,
  RDL_ERR_CUDA = -3,
  RDL_ERR_TIMEOUT = -4,
  RDL_ERR_WORKSPACE = -5,
  RDL_ERR_DEVICE_CHECK = -6,
  RDL_ERR_SCRATCH_LIMIT = -7
} rdl_status;

typedef enum { RDL_BF16 = 0, RDL_F32 = 1 } rdl_dtype;

/* flags */
#define RDL_FLAG_MEAN_SUMMARY 0x1 /* summary = mean of the 63 content keys (Table 6 ablation) */
#define RDL_FLAG_CHECKS 0x2       /* device-side index/position checks into the status word */
/* Summary layout for decode blocks: rdl_summary_pool writes, and rdl_route_score_topk reads,
 * each summary row as d bf16 "hi" terms followed by d bf16 "lo" terms (s = hi + lo to about
 * 2^-17 relative; the same 4d bytes as the fp32 row).  The split is then done once when the
 * block's summaries are pooled instead of on every decode step.  rdl_route_score_topk accepts
 * it for decode-block shapes (bf16, d = 128, at most 64 rows) and returns
 * RDL_ERR_UNSUPPORTED otherwise. */
#define RDL_FLAG_SPLIT_SUMMARY 0x4
/* Test only: the failure path of a bounded wait.  With this flag the prefill selected-chunk
 * kernel of rdl_route_attn (either of its two forms) waits, with a short limit, on a barrier
 * nothing arrives on, once its first K/V slab and query loads are in flight.  The wait runs out: the
 * kernel records RDL_ERR_TIMEOUT, every role stops, the copies and MMAs in flight drain, tensor
 * memory is freed and the kernel returns; the call's outputs are then not valid.  Nothing
 * faults and the context stays usable (the next call without the flag computes normally). */
#define RDL_FLAG_WAIT_TEST 0x8

#define RDL_CHUNK 64

typedef struct {
  int B;        /* batch */
  int L;        /* sequence / cache length, multiple of 64 */
  int Lq;       /* query rows */
  int Hq;       /* query heads */
  int Hkv;      /* KV heads; Hq % Hkv == 0 */
  int d;        /* head dim: 64 or 128 */
  int D;        /* hidden size of x (residual input) */
  int r;        /* residual rank, 1..128 (0: no residual) */
  int K;        /* selected chunks per query, 1..min(C, 64) */
  int w;        /* local-window radius; < 0: no window */
  float lambda; /* entropy weight of the route score */
  int flags;    /* RDL_FLAG_* */
} rdl_dims;

/* Which workspace a call needs (rdl_workspace_bytes). */
#define RDL_WS_SCORE 0
#define RDL_WS_ATTN 1
#define RDL_WS_SWA 2

/*
 * rdl_summary_pool -- summary key, pooling entropy and mask-slot output of every chunk
 * (Figure 3 caption: "Its query pools the content keys with an intra-chunk softmax, and
 * the weighted sum is the summary key s_c"; the entropy of those weights is the second
 * routing signal, "The 172x Speedup Has an Evidence Budget", same section).
 *
 * For b, head h, chunk c:  l_j = tau * q_mask[b,c,h] . k[b,g(h),64c+j],  j = 0..62;
 *   a = softmax(l);  summary[b,h,c] = sum_j a_j k_j;  entropy[b,h,c] = -sum_j a_j ln a_j;
 *   o_mask row (c, h) = sum_j a_j v[b,g(h),64c+j]          (only when v and o_mask are set)
 * With RDL_FLAG_MEAN_SUMMARY, a_j = 1/63.
 *
 * q_mask: the query row of chunk c's mask slot is at q_mask + b*q_batch_stride +
 *   c*q_chunk_stride (element strides; the row holds Hq*d elements).  For a full-sequence
 *   q [B, L, Hq, d] pass q + 63*Hq*d, q_chunk_stride = 64*Hq*d, q_batch_stride = L*Hq*d.
 * o_mask (nullable): written with the same strides as q_mask, in the storage dtype.
 * v (nullable): needed only when o_mask is set.  Lq, D, r, K, w, lambda are ignored.
 */
rdl_status rdl_summary_pool(const void* q_mask, long long q_chunk_stride,
                            long long q_batch_stride, const void* k, const void* v,
                            const rdl_dims* dims, rdl_dtype dtype, float* summary,
                            float* entropy, void* o_mask, void* stream);

/*
 * rdl_route_score_topk -- routing residual, route score, GQA group max and per-query
 * top-K (Figure 3 caption: "A content query adds a low-rank residual and scores these
 * summaries.  Inside a GQA group the scores are reduced by a maximum, and the top K
 * chunks are shared by every head in the group"; remote chunks only, Table 3).
 *
 * For a content row i at position p:
 *   q_res[h] = q[b,i,h] + ((x[b,i] W_down) W_up)[h*d : h*d+d]
 *   z[h,c]   = tau * q_res[h] . summary[b,h,c] - lambda * entropy[b,h,c]   for c in E(p)
 *   zeta[g,c] = max over h in group g of z[h,c]
 *   T(i,g)   = the K eligible chunks with largest zeta (ties: smaller chunk index first);
 *              fewer than K eligible: the rest of idx is -1.
 * Outputs idx (ascending chunk order) and z_sel (z of each selected chunk, per head).
 * Mask-slot rows: idx = -1, z_sel = -inf.  r = 0 or x == NULL: no residual.
 * workspace: device scratch of at least rdl_workspace_bytes(RDL_WS_SCORE, dims, dtype)
 *   bytes, 256-byte aligned (RDL_ERR_WORKSPACE if smaller).
 */
rdl_status rdl_route_score_topk(const void* q, const int32_t* q_pos, const void* x,
                                const void* w_down, const void* w_up, const float* summary,
                                const float* entropy, const rdl_dims* dims, rdl_dtype dtype,
                                int32_t* idx, float* z_sel, void* workspace,
                                size_t ws_bytes, void* stream);

/*
 * rdl_route_attn -- two-level partitioned attention of the route layer (Figure 3
 * caption: "Attention mass puts the selected chunk scores and the local-window
 * log-sum-exp in one partition, then a second softmax distributes each chunk's mass over
 * its content tokens").
 *
 * For a content row i at position p, head h, group g:
 *   lambda_loc = LSE_{j in W(p)} tau q.k_j,  o_loc = softmax-weighted sum of v_j over W(p)
 *   for c in T(i,g):  o_c = softmax over content(c) of tau q.k_j, applied to v_j
 *   Z = e^lambda_loc + sum_c e^{z_sel[c]};  o = (e^lambda_loc o_loc + sum_c e^{z_sel[c]} o_c)/Z
 *   lse = ln Z  (lse nullable).
 * idx entries must be -1 or in [0, C) and must not touch W(p) (as produced by
 * rdl_route_score_topk); with RDL_FLAG_CHECKS a violation is recorded in the status word
 * and the entry is skipped.
 * workspace: at least rdl_workspace_bytes(RDL_WS_ATTN, dims, dtype) bytes.
 */
rdl_status rdl_route_attn(const void* q, const int32_t* q_pos, const void* k, const void* v,
                          const int32_t* idx, const float* z_sel, const rdl_dims* dims,
                          rdl_dtype dtype, void* o, float* lse, void* workspace,
                          size_t ws_bytes, void* stream);

/*
 * rdl_route_attn_noalloc -- rdl_route_attn for callers that cannot allocate device memory.
 * The paper has no counterpart to this call: it exists for deployment.  Some hosts give a
 * kernel library no way to obtain scratch memory at call time -- inference engines that
 * plan every device buffer before serving and forbid allocation on the request path (a
 * cudaMalloc there synchronises the device and can fail once memory is fragmented), and
 * plugin interfaces that hand the plugin its inputs and outputs but no allocator.  This
 * entry point takes the same arguments as rdl_route_attn minus the workspace and uses a
 * static scratch array that librdl.so itself holds in device memory instead.
 *
 * Scratch limit: RDL_NOALLOC_SCRATCH_BYTES (32 MiB) per device, reserved on every GPU
 * that loads the library, until the process exits.  A call whose
 * rdl_workspace_bytes(RDL_WS_ATTN, dims, dtype) exceeds it returns RDL_ERR_SCRATCH_LIMIT
 * and launches nothing (a 32-query decode block over 28 heads with K = 32 and a +-256 window
 * needs about 14.5 MiB).
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current); make that first call before any stream capture begins.  The
 * address is kept per device and context: after cudaDeviceReset the next call on that
 * device looks it up again (again before any capture).
 * Nothing here calls cudaMalloc, cudaFree or any allocating routine.
 * Every call on a device shares the one array and leaves its contents behind; no part of
 * it needs to start at zero.  Calls issued one after another on one stream are safe (each
 * call's kernels wait for the previous call's last reads of the array before writing it).
 * Calls that overlap on the GPU (concurrent streams, or several host threads on different
 * streams) race on the array: serialise them.
 */
#define RDL_NOALLOC_SCRATCH_BYTES (32u << 20)
rdl_status rdl_route_attn_noalloc(const void* q, const int32_t* q_pos, const void* k,
                                  const void* v, const int32_t* idx, const float* z_sel,
                                  const rdl_dims* dims, rdl_dtype dtype, void* o, float* lse,
                                  void* stream);

/*
 * rdl_swa_attn -- bidirectional sliding-window attention of the non-route layers
 * ("on every fourth layer ... the other layers use a bidirectional sliding window",
 * abstract; radius per Table 3).  Every row, mask slots included:
 *   o = softmax_{j in W(p)} (tau q.k_j) applied to v_j,   lse = LSE (nullable).
 * Requires w >= 0.  K, D, r, lambda are ignored.
 * workspace (nullable): rdl_workspace_bytes(RDL_WS_SWA, dims, dtype) bytes, 256-byte
 *   aligned.  It is nonzero only for few query rows (decode blocks), where the window's
 *   keys are split across CTAs; with NULL the unsplit (slower for few rows) path runs.
 */
rdl_status rdl_swa_attn(const void* q, const int32_t* q_pos, const void* k, const void* v,
                        const rdl_dims* dims, rdl_dtype dtype, void* o, float* lse,
                        void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes a call needs (0 if none); 0 also for invalid dims. */
size_t rdl_workspace_bytes(int which, const rdl_dims* dims, rdl_dtype dtype);

/* Synchronises `stream`, returns and clears the device status word: RDL_OK,
 * RDL_ERR_DEVICE_CHECK (a RDL_FLAG_CHECKS check failed) or RDL_ERR_TIMEOUT (a bounded
 * wait ran out); RDL_ERR_CUDA if the stream reports an error. */
rdl_status rdl_last_device_status(void* stream);

/* Static description of a status code. */
const char* rdl_status_string(rdl_status s);

/* Number of kernels this library has launched in this process (all devices, all
 * threads); a diagnostic for counting launches inside a timed region. */
unsigned long long rdl_launch_count(void);

/* Library version, "major.minor.patch". */
const char* rdl_version(void);

#ifdef __cplusplus
}
#endif
#endif /* RDL_H */
