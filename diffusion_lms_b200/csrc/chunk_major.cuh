// Selected-chunk attention of the route layer for prefills, chunk-major over the whole sequence
// (Prefilling-dLLM v2, Figure 3 caption: "Attention mass puts the selected chunk scores and the
// local-window log-sum-exp in one partition, then a second softmax distributes each chunk's mass
// over its content tokens").
//
// A query row's chunks are its own top-K, so for long sequences the rows that share a chunk are
// scattered over the whole sequence: a chunk of a group is selected by about K * 64 rows at any
// length.  The path therefore works chunk by chunk over all rows:
//
//   cm_count_kernel    per (batch, group) and chunk, the number of (row, slot) selections
//                      (shared-memory histograms of row blocks, then one atomic per bin);
//   cm_scan_kernel     chunk offsets of the buckets, and the work items: each bucket cut into
//                      pieces of at most CM_IT entries;
//   cm_scatter_kernel  every selection (row << 6 | slot) into its chunk's bucket (the order
//                      inside a bucket does not matter: every output row is computed alone);
//   cm_attn_kernel     persistent CTAs over the work items.  An item's K/V slab lands once by
//                      TMA; its entries are processed 16 at a time ("passes": M = 128 rows =
//                      16 queries x 8 head slots, query rows gathered by TMA):
//                        S = Q K_c^T   tcgen05.mma M=128 N=64 K=128      (tensor memory)
//                        P = softmax of S over the chunk's 63 content keys   (bf16, smem)
//                        O = P V_c     tcgen05.mma M=128 N=128 K=64      (tensor memory)
//                      and each (row, slot, head) output o_c is stored in fp16;
//   cm_combine_kernel  per (row, head): M = max(window lse, z_c), Z = e^{lse_w - M} + sum_c
//                      e^{z_c - M}, o = (e^{lse_w - M} o_w + sum_c e^{z_c - M} o_c) / Z, lse = ln Z.
//
// Warp roles of cm_attn_kernel (384 threads): warp 0 walks the items and loads K/V (TMA, one
// lane), warp 1 issues the MMAs (warp-collective), warp 2 gathers the query rows of a pass (one
// TMA box of 8 head slots per entry, lanes 0-15), warps 4-7 the softmax (TMEM lane quarter =
// warp % 4, one row per thread), warps 8-11 the epilogue (same lane mapping).  Tensor memory: S in two buffers of 64 columns, O in two of
// 128.  Shared memory: two K/V stages of 32 KB, two Q tiles of 32 KB (token-major, 2 KB per
// query: its 8 head rows for columns 0-63, then 64-127), two P tiles of 16 KB; 128-byte swizzle.
// Every wait is bounded; after a timeout the kernel records RDL_ERR_TIMEOUT, every role stops,
// the MMAs in flight drain, the last TMA loads land and tensor memory is freed.
#pragma once
#include "common.cuh"
#include "tc.cuh"

namespace rdl {

constexpr int CM_IT = 128;                 // entries per work item (8 passes)
constexpr int CM_PQ = 16;                  // queries per pass
constexpr int CM_THREADS = 12 * 32;
constexpr int CM_ROWS = 512;               // rows per CTA of the bucketing kernels
constexpr int CM_MAXC = 8192;
constexpr int CM_OFF_KV = 0;               // stage s at 32 KB s: K, V at + 16 KB
constexpr int CM_OFF_Q = 65536;            // buffer b at + 32 KB b
constexpr int CM_OFF_P = CM_OFF_Q + 65536; // buffer b at + 16 KB b
constexpr int CM_OFF_LIST = CM_OFF_P + 32768;     // the item's entries [CM_IT] int
constexpr int CM_OFF_BAR = CM_OFF_LIST + CM_IT * 4;
constexpr int CM_SMEM = CM_OFF_BAR + 256 + 1024;
static_assert(CM_SMEM <= 227 * 1024, "shared memory");

struct CmItem {
  int bg, c, start, n;                     // (batch x groups + group), chunk, bucket range
};

// the selection (row at position p, slot value c) as a chunk of the path, -1 if it is not
// one: an index outside [0, C) is skipped, and with RDL_FLAG_CHECKS so is one touching the
// window; with `record` both are recorded in the status word
__device__ __forceinline__ int cm_entry_chunk(int c, int p, int C, int w, int flags, bool record) {
  if (c < 0 || is_mask_slot(p)) return -1;
  const bool checks = (flags & RDL_FLAG_CHECKS) != 0;
  if (c >= C || (checks && !chunk_eligible(c, p, w))) {
    if (checks && record) record_status(RDL_ERR_DEVICE_CHECK);
    return -1;
  }
  return c;
}

// ------------------------------------------------------------------ bucketing
// grid (ceil(Lq / CM_ROWS), B * Hkv), 512 threads; counts [B*Hkv][C]
__global__ void __launch_bounds__(512) cm_count_kernel(const int32_t* __restrict__ idx,
                                                       const int32_t* __restrict__ q_pos, int Lq, int L,
                                                       int Hkv, int K, int w, int flags,
                                                       int* __restrict__ counts) {
  extern __shared__ int cm_hist[];
  const int C = L / S, bg = blockIdx.y, b = bg / Hkv;
  const int r0 = blockIdx.x * CM_ROWS, r1 = min(Lq, r0 + CM_ROWS);
  for (int c = threadIdx.x; c < C; c += blockDim.x) cm_hist[c] = 0;
  __syncthreads();
  const int32_t* ib = idx + (size_t)bg * Lq * K;
  for (int e = r0 * K + threadIdx.x; e < r1 * K; e += blockDim.x) {
    const int i = e / K;
    const int p = q_pos ? q_pos[(size_t)b * Lq + i] : i;
    const int c = cm_entry_chunk(ib[e], p, C, w, flags, true);
    if (c >= 0) atomicAdd(&cm_hist[c], 1);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x)
    if (cm_hist[c]) atomicAdd(&counts[(size_t)bg * C + c], cm_hist[c]);
}

// grid (B * Hkv), 1024 threads: offs = exclusive scan of counts; items of each bucket appended
// at a position taken from the global item counter
__global__ void __launch_bounds__(1024) cm_scan_kernel(const int* __restrict__ counts, int C,
                                                       int* __restrict__ offs, int* __restrict__ nitems,
                                                       CmItem* __restrict__ items) {
  __shared__ int ws[2 * 32];
  __shared__ int base_s;
  const int bg = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (C + 1023) / 1024, c0 = min(C, tid * per), c1 = min(C, c0 + per);
  const int* cnt = counts + (size_t)bg * C;
  int le = 0, li = 0;
  for (int c = c0; c < c1; ++c) {
    le += cnt[c];
    li += (cnt[c] + CM_IT - 1) / CM_IT;
  }
  int se = le, si = li;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, se, o), bb = __shfl_up_sync(0xffffffffu, si, o);
    if (lane >= o) {
      se += a;
      si += bb;
    }
  }
  if (lane == 31) {
    ws[2 * warp] = se;
    ws[2 * warp + 1] = si;
  }
  __syncthreads();
  int be = 0, bi = 0, ti = 0;
  for (int x = 0; x < 32; ++x) {
    if (x < warp) {
      be += ws[2 * x];
      bi += ws[2 * x + 1];
    }
    ti += ws[2 * x + 1];
  }
  if (tid == 0) base_s = atomicAdd(nitems, ti);
  __syncthreads();
  int oe = be + se - le, oi = base_s + bi + si - li;   // bucket offsets within the group's list
  for (int c = c0; c < c1; ++c) {
    const int n = cnt[c];
    offs[(size_t)bg * C + c] = oe;
    for (int s0 = 0; s0 < n; s0 += CM_IT) items[oi++] = CmItem{bg, c, oe + s0, min(CM_IT, n - s0)};
    oe += n;
  }
}

// grid as cm_count_kernel; list [B*Hkv][Lq*K]: entries row << 6 | slot, bucket by bucket
__global__ void __launch_bounds__(512) cm_scatter_kernel(const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ q_pos, int Lq, int L,
                                                         int Hkv, int K, int w, int flags,
                                                         const int* __restrict__ offs, int* __restrict__ cursor,
                                                         int* __restrict__ list) {
  extern __shared__ int cm_hist[];          // [C] counts, then [C] bases
  const int C = L / S, bg = blockIdx.y, b = bg / Hkv;
  int* cbase = cm_hist + C;
  const int r0 = blockIdx.x * CM_ROWS, r1 = min(Lq, r0 + CM_ROWS);
  for (int c = threadIdx.x; c < C; c += blockDim.x) cm_hist[c] = 0;
  __syncthreads();
  const int32_t* ib = idx + (size_t)bg * Lq * K;
  for (int e = r0 * K + threadIdx.x; e < r1 * K; e += blockDim.x) {
    const int i = e / K;
    const int p = q_pos ? q_pos[(size_t)b * Lq + i] : i;
    const int c = cm_entry_chunk(ib[e], p, C, w, flags, false);   // recorded by cm_count_kernel
    if (c >= 0) atomicAdd(&cm_hist[c], 1);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const int n = cm_hist[c];
    cbase[c] = n ? offs[(size_t)bg * C + c] + atomicAdd(&cursor[(size_t)bg * C + c], n) : 0;
    cm_hist[c] = 0;
  }
  __syncthreads();
  int* lb = list + (size_t)bg * Lq * K;
  for (int e = r0 * K + threadIdx.x; e < r1 * K; e += blockDim.x) {
    const int i = e / K;
    const int p = q_pos ? q_pos[(size_t)b * Lq + i] : i;
    const int c = cm_entry_chunk(ib[e], p, C, w, flags, false);
    if (c >= 0) lb[cbase[c] + atomicAdd(&cm_hist[c], 1)] = (i << 6) | (e % K);
  }
}

// ------------------------------------------------------------------ attention
struct CmBars {
  uint64_t *kvfull, *kvempty, *qfull, *qempty, *sfull, *sempty, *pfull, *pempty, *ofull, *oempty, *mdone;
  uint64_t* never;     // nothing arrives on it (RDL_FLAG_WAIT_TEST)
};
constexpr unsigned CM_TEST_POLLS = 1u << 12;   // bound of the RDL_FLAG_WAIT_TEST wait

__global__ void __launch_bounds__(CM_THREADS, 1)
    cm_attn_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                   const __grid_constant__ CUtensorMap qmap, const CmItem* __restrict__ items,
                   const int* __restrict__ nitems_p, const int* __restrict__ list, int Lq, int L, int Hq,
                   int Hkv, int K, int flags, __half* __restrict__ part) {
  constexpr int D = 128;
  extern __shared__ unsigned char cm_raw[];
  unsigned char* sm = cm_raw + ((1024u - (smem_u32(cm_raw) & 1023u)) & 1023u);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + CM_OFF_BAR);
  CmBars B{bar, bar + 2, bar + 4, bar + 6, bar + 8, bar + 10, bar + 12, bar + 14, bar + 16, bar + 18, bar + 20,
           bar + 21};
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 22);
  volatile int* abort_f = reinterpret_cast<volatile int*>(tslot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = Hq / Hkv;
  const int nitems = *nitems_p;

  if (tid == 0) {
    for (int j = 0; j < 2; ++j) {
      tc::mbar_init(&B.kvfull[j], 1);
      tc::mbar_init(&B.kvempty[j], 1);
      tc::mbar_init(&B.qfull[j], 1);
      tc::mbar_init(&B.qempty[j], 1);
      tc::mbar_init(&B.sfull[j], 1);
      tc::mbar_init(&B.sempty[j], 4);
      tc::mbar_init(&B.pfull[j], 4);
      tc::mbar_init(&B.pempty[j], 1);
      tc::mbar_init(&B.ofull[j], 1);
      tc::mbar_init(&B.oempty[j], 4);
    }
    tc::mbar_init(B.mdone, 1);
    tc::mbar_init(B.never, 1);
    *abort_f = 0;
    tc::mbar_fence_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tslot, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tslot;
  auto wait = [&](uint64_t* b_, unsigned ph) -> bool {
    for (unsigned it = 0; it < tc::kSpinLimit; ++it) {
      if (tc::mbar_try_wait(b_, ph)) return true;
      if ((it & 255u) == 255u && *abort_f) return false;
    }
    record_status(RDL_ERR_TIMEOUT);
    *abort_f = 1;
    return false;
  };

  if (warp == 0) {
    // ---------------- K/V producer: one slab pair per item, two stages
    if (lane == 0) {
      int j = 0;
      for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++j) {
        const CmItem ci = items[it];
        const int st = j & 1;
        if (j >= 2 && !wait(&B.kvempty[st], (unsigned)((j >> 1) - 1) & 1u)) break;
        unsigned char* kv = sm + CM_OFF_KV + st * 32768;
        const int krow = ci.bg * L + ci.c * S;
        tc::mbar_arrive_expect_tx(&B.kvfull[st], 32768u);
        tc::tma_load_3d(kv, &kmap, 0, krow, 0, &B.kvfull[st]);
        tc::tma_load_3d(kv + 16384, &vmap, 0, krow, 0, &B.kvfull[st]);
      }
      // the last load of each stage has landed before the CTA may exit
      for (int x = max(0, j - 2); x < j; ++x) (void)tc::mbar_wait(&B.kvfull[x & 1], (unsigned)(x >> 1) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer: S of pass k, then PV of pass k - 1
    const uint32_t idesc_s = tc::idesc_bf16(128, 64, false, false);
    const uint32_t idesc_pv = tc::idesc_bf16(128, 128, false, true);
    const uint32_t sbase = smem_u32(sm);
    bool ok = true, issued = false;
    int k = 0, j = 0;
    int pend_k = -1, pend_st = 0;       // pass whose PV is pending, its K/V stage
    bool pend_last = false;             // ... and whether it is its item's last pass
    auto issue_pv = [&]() -> bool {
      const int pb = pend_k & 1;
      const unsigned ph = (unsigned)(pend_k >> 1) & 1u;
      const bool w_ok = wait(&B.pfull[pb], ph) && wait(&B.oempty[pb], ph ^ 1u);
      if (!__all_sync(0xffffffffu, w_ok)) return false;
      tc::tc_fence_after();
      const uint64_t dP = tc::sdesc(sbase + CM_OFF_P + pb * 16384, 16, 1024);
      const uint64_t dV = tc::sdesc(sbase + CM_OFF_KV + pend_st * 32768 + 16384, 8192, 1024);
      const uint32_t dO = tbase + 128u + (uint32_t)(pb * 128);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc::mma_bf16_ss_warp(dO, dP + (uint64_t)(2 * ks), dV + (uint64_t)(128 * ks), idesc_pv, ks > 0);
      tc::mma_commit_warp(&B.ofull[pb]);
      tc::mma_commit_warp(&B.pempty[pb]);
      if (pend_last) tc::mma_commit_warp(&B.kvempty[pend_st]);
      pend_k = -1;
      return true;
    };
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++j) {
      const int n = items[it].n, st = j & 1;
      if (!__all_sync(0xffffffffu, wait(&B.kvfull[st], (unsigned)(j >> 1) & 1u))) { ok = false; break; }
      if ((flags & RDL_FLAG_WAIT_TEST) && j == 0) {
        // a wait on a barrier nothing arrives on runs out: the failure path of every wait
        bool got = false;
        for (unsigned x = 0; x < CM_TEST_POLLS && !got; ++x) got = tc::mbar_try_wait(B.never, 0);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) {
            record_status(RDL_ERR_TIMEOUT);
            *abort_f = 1;
          }
          ok = false;
          break;
        }
      }
      const uint64_t dK = tc::sdesc(sbase + CM_OFF_KV + st * 32768, 16, 1024);
      const int npass = (n + CM_PQ - 1) / CM_PQ;
      for (int p = 0; p < npass; ++p, ++k) {
        const int qb = k & 1;
        const unsigned ph = (unsigned)(k >> 1) & 1u;
        const bool w_ok = wait(&B.qfull[qb], ph) && wait(&B.sempty[qb], ph ^ 1u);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t dQ = tc::sdesc(sbase + CM_OFF_Q + qb * 32768, 16, 2048);
        const uint32_t dS = tbase + (uint32_t)(qb * 64);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc::mma_bf16_ss_warp(dS, dQ + (uint64_t)((ks >> 2) * 64 + (ks & 3) * 2),
                               dK + (uint64_t)((ks >> 2) * 512 + (ks & 3) * 2), idesc_s, ks > 0);
        tc::mma_commit_warp(&B.sfull[qb]);
        tc::mma_commit_warp(&B.qempty[qb]);
        issued = true;
        if (pend_k >= 0 && !issue_pv()) { ok = false; break; }
        pend_k = k;
        pend_st = st;
        pend_last = p + 1 == npass;
      }
    }
    if (ok && pend_k >= 0) ok = issue_pv();
    if (!ok && lane == 0) *abort_f = 1;
    if (issued) tc::mma_commit_warp(B.mdone); else tc::mbar_arrive_warp(B.mdone);
    (void)tc::mbar_wait(B.mdone, 0);       // bounded; every MMA issued has completed
    __syncwarp();
  } else if (warp == 2) {
    // ---------------- query gather: one TMA box per entry (its 8 head slots, 2 KB), issued by
    // lanes 0-15; the item's entries are staged in shared memory first
    int* lsm = reinterpret_cast<int*>(sm + CM_OFF_LIST);
    int k = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const CmItem ci = items[it];
      const int g = ci.bg % Hkv, b = ci.bg / Hkv;
      const int* lb = list + (size_t)ci.bg * Lq * K + ci.start;
      __syncwarp();
      for (int e = lane; e < ci.n; e += 32) lsm[e] = __ldcg(lb + e);
      __syncwarp();
      for (int p0 = 0; p0 < ci.n; p0 += CM_PQ, ++k) {
        const int qb = k & 1;
        if (!__all_sync(0xffffffffu, wait(&B.qempty[qb], ((unsigned)(k >> 1) & 1u) ^ 1u))) { ok = false; break; }
        const int ne = min(CM_PQ, ci.n - p0);
        if (lane == 0) tc::mbar_arrive_expect_tx(&B.qfull[qb], (unsigned)(ne * 2048));
        __syncwarp();
        if (lane < ne) {
          const int i = lsm[p0 + lane] >> 6;
          tc::tma_load_4d(sm + CM_OFF_Q + qb * 32768 + lane * 2048, &qmap, 0, g * G, 0, b * Lq + i, &B.qfull[qb]);
        }
      }
    }
    // the last loads issued into each buffer have landed before the CTA may exit
    if (lane == 0)
      for (int x = max(0, k - 2); x < k; ++x) (void)tc::mbar_wait(&B.qfull[x & 1], (unsigned)(x >> 1) & 1u);
    __syncwarp();
  } else if (warp >= 4 && warp <= 7) {
    // ---------------- softmax: row r = (entry r / 8, head slot r % 8), 64 keys per row
    const int quad = warp & 3, r = 32 * quad + lane;
    const float sl2 = rsqrtf((float)D) * LOG2E;
    const uint32_t lrow = tc::taddr(tbase, 32 * quad, 0);
    int k = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const int n = items[it].n;
      for (int p0 = 0; p0 < n; p0 += CM_PQ, ++k) {
        const int sb = k & 1;
        const unsigned ph = (unsigned)(k >> 1) & 1u;
        if (!wait(&B.sfull[sb], ph)) { ok = false; break; }
        tc::tc_fence_after();
        float v[64];
        tc::tmem_ld32(lrow + (uint32_t)(sb * 64), v);
        tc::tmem_ld32(lrow + (uint32_t)(sb * 64 + 32), v + 32);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&B.sempty[sb]);
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < CONTENT; ++e) mx = fmaxf(mx, v[e]);
        const float off = mx * sl2;
        float l = 0.f;
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          v[e] = e < CONTENT ? fast_exp2(fmaf(v[e], sl2, -off)) : 0.f;
          l += v[e];
        }
        const float inv = 1.f / l;
        if (!wait(&B.pempty[sb], ph ^ 1u)) { ok = false; break; }
        unsigned char* prow = sm + CM_OFF_P + sb * 16384 + r * 128;
#pragma unroll
        for (int uu = 0; uu < 8; ++uu) {
          const uint4 pk = make_uint4(pack_bf16(v[8 * uu] * inv, v[8 * uu + 1] * inv),
                                      pack_bf16(v[8 * uu + 2] * inv, v[8 * uu + 3] * inv),
                                      pack_bf16(v[8 * uu + 4] * inv, v[8 * uu + 5] * inv),
                                      pack_bf16(v[8 * uu + 6] * inv, v[8 * uu + 7] * inv));
          *reinterpret_cast<uint4*>(prow + ((uu ^ (r & 7)) << 4)) = pk;
        }
        tc::fence_proxy_async();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&B.pfull[sb]);
      }
    }
  } else if (warp >= 8) {
    // ---------------- epilogue: O row (entry, head slot) -> fp16 partial of (row, slot, head)
    const int quad = warp & 3, r = 32 * quad + lane, m = r >> 3, hs = r & 7;
    const uint32_t lrow = tc::taddr(tbase, 32 * quad, 128);
    int k = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const CmItem ci = items[it];
      const int* lb = list + (size_t)ci.bg * Lq * K + ci.start;
      for (int p0 = 0; p0 < ci.n; p0 += CM_PQ, ++k) {
        const int ob = k & 1;
        const bool valid = p0 + m < ci.n && hs < G;
        const int en = valid ? __ldcg(lb + p0 + m) : 0;
        if (!wait(&B.ofull[ob], (unsigned)(k >> 1) & 1u)) { ok = false; break; }
        tc::tc_fence_after();
        __half* dst = part + (((size_t)ci.bg * Lq + (en >> 6)) * K + (en & 63)) * (size_t)(G * D) + hs * D;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float v[64];
          tc::tmem_ld32(lrow + (uint32_t)(ob * 128 + 64 * hf), v);
          tc::tmem_ld32(lrow + (uint32_t)(ob * 128 + 64 * hf + 32), v + 32);
          tc::tmem_wait_ld();
          if (hf == 1) {
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&B.oempty[ob]);
          }
          if (valid) {
#pragma unroll
            for (int uu = 0; uu < 8; ++uu) {
              const __half2 a0 = __floats2half2_rn(v[8 * uu], v[8 * uu + 1]);
              const __half2 a1 = __floats2half2_rn(v[8 * uu + 2], v[8 * uu + 3]);
              const __half2 a2 = __floats2half2_rn(v[8 * uu + 4], v[8 * uu + 5]);
              const __half2 a3 = __floats2half2_rn(v[8 * uu + 6], v[8 * uu + 7]);
              uint4 pk;
              pk.x = *reinterpret_cast<const uint32_t*>(&a0);
              pk.y = *reinterpret_cast<const uint32_t*>(&a1);
              pk.z = *reinterpret_cast<const uint32_t*>(&a2);
              pk.w = *reinterpret_cast<const uint32_t*>(&a3);
              __stcg(reinterpret_cast<uint4*>(dst + 64 * hf) + uu, pk);
            }
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tbase, 512);
  }
}

// ------------------------------------------------------------------ combine
// One warp per (b, i, h); lane l owns head dims 4l .. 4l+3.  Window part: nsw key-split
// planes of (lse, normalised output); chunk parts: the fp16 partials of cm_attn_kernel.
constexpr int CM_COMB_WARPS = 4;
__global__ void __launch_bounds__(CM_COMB_WARPS * 32, 3) cm_combine_kernel(const int32_t* __restrict__ q_pos,
                                                         const int32_t* __restrict__ idx,
                                                         const float* __restrict__ z_sel,
                                                         const __half* __restrict__ part,
                                                         const float* __restrict__ o_loc,
                                                         const float* __restrict__ lam_loc, int nsw, int B,
                                                         int L, int Lq, int Hq, int Hkv, int K, int w,
                                                         int flags, __nv_bfloat16* __restrict__ o,
                                                         float* __restrict__ lse) {
  constexpr int D = 128;
  const int lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * CM_COMB_WARPS + (threadIdx.x >> 5);
  if (item >= (long long)B * Lq * Hq) return;
  const int h = (int)(item % Hq);
  const int i = (int)((item / Hq) % Lq);
  const int b = (int)(item / ((long long)Hq * Lq));
  const int C = L / S, G = Hq / Hkv, g = h / G, hl = h % G;
  const int p = q_pos ? q_pos[(size_t)b * Lq + i] : i;
  if (is_mask_slot(p)) return;
  const size_t rh = (size_t)(b * Lq + i) * Hq + h;
  const size_t li = (size_t)(b * Hq + h) * Lq + i;
  const size_t plane_l = (size_t)B * Hq * Lq, plane_o = (size_t)B * Lq * Hq * D;
  const size_t bg = (size_t)b * Hkv + g;
  // Every load that does not depend on a weight is issued first, so the row costs one memory
  // round trip: the chunk ids and logits (lanes k, k + 32 hold slot k), the first window
  // plane, and the chunk outputs of slots 0-31 (a slot without a chunk is read too and gets
  // weight 0).
  const int32_t* irow = idx + (bg * Lq + i) * K;
  const float* zrow = z_sel + li * K;
  int ck[2] = {-1, -1};
  float zr[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int k = lane + 32 * u;
    if (k < K) {
      ck[u] = irow[k];
      zr[u] = zrow[k];
    }
  }
  const float ls0 = nsw > 0 ? lam_loc[li] : -INFINITY;
  const float4 vw0 = nsw > 0 ? *reinterpret_cast<const float4*>(o_loc + rh * D + 4 * lane)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
  const __half* pb = part + ((bg * Lq + i) * K * G + hl) * D + 4 * lane;
  uint2 raw[32];
#pragma unroll
  for (int u = 0; u < 32; ++u)
    raw[u] = u < K ? __ldcs(reinterpret_cast<const uint2*>(pb + (size_t)u * G * D)) : make_uint2(0u, 0u);
  float zk[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    // the same rule as the bucketing kernels (no status recorded a second time)
    const int c = ck[u];
    bool on = c >= 0 && c < C;
    if (on && (flags & RDL_FLAG_CHECKS) && !chunk_eligible(c, p, w)) on = false;
    if (on) zk[u] = zr[u];
  }
  float M = warp_max(fmaxf(zk[0], zk[1]));
  M = fmaxf(M, ls0);
  for (int sw = 1; sw < nsw; ++sw) M = fmaxf(M, lam_loc[sw * plane_l + li]);
  if (M == -INFINITY) M = 0.f;
  const float ek0 = zk[0] == -INFINITY ? 0.f : expf(zk[0] - M);
  const float ek1 = zk[1] == -INFINITY ? 0.f : expf(zk[1] - M);
  float Z = warp_sum(ek0 + ek1);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sw = 0; sw < nsw; ++sw) {
    const float ls = sw == 0 ? ls0 : lam_loc[sw * plane_l + li];
    if (ls == -INFINITY) continue;
    const float f = expf(ls - M);
    Z += f;
    const float4 vw = sw == 0 ? vw0 : *reinterpret_cast<const float4*>(o_loc + sw * plane_o + rh * D + 4 * lane);
    acc.x += f * vw.x; acc.y += f * vw.y; acc.z += f * vw.z; acc.w += f * vw.w;
  }
#pragma unroll
  for (int u = 0; u < 32; ++u) {
    const float f = __shfl_sync(0xffffffffu, ek0, u);
    if (u < K && f != 0.f) {
      const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw[u].x));
      const float2 c2 = __half22float2(*reinterpret_cast<const __half2*>(&raw[u].y));
      acc.x += f * a.x; acc.y += f * a.y; acc.z += f * c2.x; acc.w += f * c2.y;
    }
  }
  for (int k0 = 32; k0 < K; k0 += 8) {        // K > 32: the rest in batches of 8
    uint2 r8[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      r8[u] = k0 + u < K ? __ldcs(reinterpret_cast<const uint2*>(pb + (size_t)(k0 + u) * G * D)) : make_uint2(0u, 0u);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float f = __shfl_sync(0xffffffffu, ek1, (k0 + u) & 31);
      if (k0 + u < K && f != 0.f) {
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&r8[u].x));
        const float2 c2 = __half22float2(*reinterpret_cast<const __half2*>(&r8[u].y));
        acc.x += f * a.x; acc.y += f * a.y; acc.z += f * c2.x; acc.w += f * c2.y;
      }
    }
  }
  const float inv = Z > 0.f ? 1.f / Z : 0.f;
  __nv_bfloat16* orow = o + rh * D + 4 * lane;
  const __nv_bfloat162 o01 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  const __nv_bfloat162 o23 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&o01);
  pk.y = *reinterpret_cast<const uint32_t*>(&o23);
  *reinterpret_cast<uint2*>(orow) = pk;
  if (lse && lane == 0) lse[li] = Z > 0.f ? M + logf(Z) : -INFINITY;
}

}  // namespace rdl
