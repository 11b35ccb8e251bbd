// Selected-chunk attention of the route layer on tcgen05 tensor cores (prefill).
//
// Same partition as chunk_mma_kernel ([v2] Figure 3 caption: the selected chunk scores and
// the window's log-sum-exp share one softmax partition; a second softmax spreads each
// chunk's mass over its 63 content tokens), organised so that one load of a chunk's K/V
// serves every query of a 45-row tile that selected it:
//
//   CTA = (45 consecutive query rows, one KV group).  The tile's (row, slot) selections are
//   bucketed by chunk, each bucket in ascending row order.  For every chunk in the union,
//   in ascending order, the K/V slab (2 x 16 KB) arrives by TMA, and the rows that selected
//   it are processed 8 queries (64 rows = 8 x 8 padded heads) at a time ("passes"):
//     S   = Q_rows K_c^T        tcgen05.mma M=64 N=64 K=128 -> TMEM S region
//     P   = e^{S - max} * w_{i,h,c} / l   over the 63 content keys, written to smem (bf16)
//     T   = V_c^T P^T           tcgen05.mma M=128 (head dim) N=8*nq K=64 -> TMEM T region
//     O^T[:, 8q..8q+8) += T[:, 8j..8j+8)   lane-local TMEM adds into each query's home
//                                         columns (one thread per head-dim lane)
//   where w = e^{z_{i,h,c} - M}/Z is fixed up front (z_sel and the window lse are inputs).
//   The home accumulators O^T [128 lanes x 45*8 columns] stay in TMEM for the whole tile;
//   the epilogue adds the window part and writes o once.
//
// Costs that shape the design (measured on B200): a tcgen05.mma issued by a converged warp
// takes about the same time (~63 cycles) for every shape up to N = 128 (~144 from a
// single-lane branch), so a pass is bounded by its 12 MMAs; a
// TMA instruction takes ~130 cycles to issue whatever its box size, so loads are made as
// large as possible: K and V one 3D box each, and the Q rows of a pass one 4D box per run
// of consecutive query tokens (the buckets are sorted so that runs are long).  S and T
// have their own TMEM regions (S is released as soon as the softmax has read it), two
// softmax groups take alternate passes, and the home adds are split over 8 warps.
//
// Warp roles (640 threads):
//   warp 0        Q producer (TMA, lane 0)
//   warp 1        TMEM owner, issuer of the S MMAs (warp-collective issue)
//   warp 2        issuer of the PV MMAs (warp-collective issue)
//   warps 3-10    two softmax groups (even / odd passes), one warp per TMEM lane quarter.
//                 An M=64 result occupies lanes 0-15 of each quarter; the 16x256b load
//                 shape spreads them over all 32 threads (thread t: rows t/4 and t/4+8,
//                 columns 8i + 2(t%4) + {0,1}).
//   warps 11-18   home-column adds (heads 0-3 / 4-7), then, with warps 3-10, the epilogue.
//   warp 19       K/V producer (TMA, lane 0)
// TMEM columns: home [0, 360), S [384, 448), T [448, 512).
// Shared-memory Q tile of a pass: query slot j at j * 2 KB (columns 0-63 of its 8 head
// rows, then columns 64-127), i.e. K-major with 128-byte swizzle, SBO 2 KB.
// Every wait is bounded; on a timeout the kernel records RDL_ERR_TIMEOUT, every role
// stops, the MMAs in flight drain, TMEM is freed and the kernel returns.
#pragma once
#include "common.cuh"
#include "tc.cuh"

namespace rdl {

constexpr int CT_TQ = 45;                  // query rows per CTA (<= 64: row masks; 16K rows x 4 groups -> 9.9 waves of 148)
constexpr int CT_HP = 8;                   // rows per query in S / columns per query in TMEM
constexpr int CT_QP = 8;                   // queries per pass (M = 64)
constexpr int CT_NSLOT = 3;                // K/V ring depth
constexpr int CT_NA = 3;                   // Q ring depth
constexpr int CT_MAXC = 2048;              // chunks (L <= 131072)
constexpr int CT_MAXK = 64;
constexpr int CT_HOME = CT_TQ * CT_HP;     // 360 home columns
constexpr int CT_SCOL = 384;               // S region
constexpr int CT_TCOL = 448;               // T region
static_assert(CT_HOME <= CT_SCOL, "TMEM columns");
constexpr int CT_WARPS = 20;
constexpr int CT_THREADS = CT_WARPS * 32;
constexpr int CT_EPI_THREADS = 16 * 32;    // warps 3-18
constexpr int CT_KV_WARP = 19;

// shared-memory map (bytes from the 1024-aligned base)
constexpr int CT_OFF_KV = 0;                                   // slot s: K at s*32K, V at +16K
constexpr int CT_OFF_A = CT_OFF_KV + CT_NSLOT * 32768;         // NA x 16 KB Q tiles
constexpr int CT_OFF_P = CT_OFF_A + CT_NA * 16384;             // 2 x 8 KB P tiles
constexpr int CT_OFF_BAR = CT_OFF_P + 2 * 8192;                // mbarriers
constexpr int CT_NBAR = 2 * CT_NSLOT + 2 * CT_NA + 12;
constexpr int CT_OFF_MISC = CT_OFF_BAR + 256;                  // tmem base, abort, nunion
constexpr int CT_OFF_MASK = CT_OFF_MISC + 128;                 // row masks [MAXC] u64
constexpr int CT_OFF_OFS = CT_OFF_MASK + CT_MAXC * 8;          // bucket offsets [MAXC] int
constexpr int CT_OFF_UNI = CT_OFF_OFS + CT_MAXC * 4;           // union [MAXC] u32
constexpr int CT_OFF_ENT = CT_OFF_UNI + CT_MAXC * 4;           // entries [TQ*MAXK] u16
constexpr int CT_OFF_MW = CT_OFF_ENT + CT_TQ * CT_MAXK * 2;    // M [TQ][8]
constexpr int CT_OFF_IZ = CT_OFF_MW + CT_TQ * 8 * 4;           // 1/Z [TQ][8]
constexpr int CT_OFF_WW = CT_OFF_IZ + CT_TQ * 8 * 4;           // window mass [TQ][8]
constexpr int CT_OFF_POS = CT_OFF_WW + CT_TQ * 8 * 4;          // positions [TQ]
constexpr int CT_OFF_PART = CT_OFF_POS + CT_TQ * 4;            // scan partials [WARPS][2]
constexpr int CT_SMEM = CT_OFF_PART + CT_WARPS * 8 + 1024;     // + alignment slack
static_assert(CT_NBAR * 8 <= 256, "barrier area");
static_assert(CT_SMEM <= 227 * 1024, "shared memory");
static_assert(CT_TQ <= 64, "row masks are 64-bit");

// Tensor maps of one launch: q as runs of 1..8 consecutive tokens (make_tmap_q_run), K and V
// as 64-row slabs (make_tmap_kv_halves).
struct CtMaps {
  CUtensorMap q[8];
  CUtensorMap k, v;
};

struct CtBars {
  uint64_t* full;    // [NSLOT] K/V landed
  uint64_t* empty;   // [NSLOT] K/V slot released (one commit from each MMA thread)
  uint64_t* afull;   // [NA] Q tile landed
  uint64_t* aempty;  // [NA] Q tile consumed by the S MMAs (commit)
  uint64_t* sfull;   // [2] S of an even / odd pass ready (commit)
  uint64_t* sempty;  // S region read by the softmax group of the pass (4 arrivals)
  uint64_t* pfull;   // [2] P of an even / odd pass written (4 arrivals)
  uint64_t* pempty;  // [2] P consumed by the PV MMAs (commit)
  uint64_t* tfull;   // T ready (commit)
  uint64_t* tempty;  // T added into the home columns (8 arrivals)
  uint64_t* done;    // [2] every MMA of the S / PV issuer complete (before TMEM is freed)
  uint64_t* never;   // nothing arrives on it (RDL_FLAG_WAIT_TEST)
};
constexpr unsigned CT_TEST_POLLS = 1u << 12;   // bound of the RDL_FLAG_WAIT_TEST wait

// bounded wait that also gives up as soon as another role has aborted
__device__ __forceinline__ bool ct_wait(uint64_t* bar, unsigned parity, volatile int* abort_flag) {
  for (unsigned it = 0; it < tc::kSpinLimit; ++it) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u && *abort_flag) return false;
  }
  record_status(RDL_ERR_TIMEOUT);
  *abort_flag = 1;
  return false;
}

__device__ __forceinline__ uint32_t ct_union(int c, int start, int cnt) {
  return (uint32_t)c | ((uint32_t)start << 12) | ((uint32_t)cnt << 24);
}

__device__ __forceinline__ void ct_epi_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(CT_EPI_THREADS) : "memory");
}

__global__ void __launch_bounds__(CT_THREADS, 1) chunk_tc_kernel(
    const __grid_constant__ CtMaps maps, const int32_t* __restrict__ q_pos, const int32_t* __restrict__ idx,
    const float* __restrict__ z_sel, const float* __restrict__ o_loc, const float* __restrict__ lam_loc, int nsw,
    int L, int Lq, int Hq, int Hkv, int K, int w, int flags, __nv_bfloat16* __restrict__ o,
    float* __restrict__ lse) {
  extern __shared__ unsigned char ct_raw[];
  unsigned char* sm = ct_raw + ((1024u - (smem_u32(ct_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = Hq / Hkv, C = L / S;
  const int i0 = blockIdx.x * CT_TQ;
  const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + CT_OFF_BAR);
  uint64_t* b2 = bars + 2 * CT_NSLOT + 2 * CT_NA;
  CtBars B{bars, bars + CT_NSLOT, bars + 2 * CT_NSLOT, bars + 2 * CT_NSLOT + CT_NA,
           b2, b2 + 2, b2 + 3, b2 + 5, b2 + 7, b2 + 8, b2 + 9, b2 + 11};
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(sm + CT_OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CT_OFF_MISC + 4);
  int* nunion_s = reinterpret_cast<int*>(sm + CT_OFF_MISC + 8);
  unsigned long long* mask = reinterpret_cast<unsigned long long*>(sm + CT_OFF_MASK);
  int* ofs = reinterpret_cast<int*>(sm + CT_OFF_OFS);
  uint32_t* uni = reinterpret_cast<uint32_t*>(sm + CT_OFF_UNI);
  uint16_t* ent = reinterpret_cast<uint16_t*>(sm + CT_OFF_ENT);
  float* Mw = reinterpret_cast<float*>(sm + CT_OFF_MW);
  float* iZ = reinterpret_cast<float*>(sm + CT_OFF_IZ);
  float* Ww = reinterpret_cast<float*>(sm + CT_OFF_WW);
  int* posv = reinterpret_cast<int*>(sm + CT_OFF_POS);
  int* part = reinterpret_cast<int*>(sm + CT_OFF_PART);

  // ---------------------------------------------------------------- set-up
  if (warp == 1) {
    tc::tmem_alloc(tmem_s, 512);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int j = 0; j < CT_NSLOT; ++j) { tc::mbar_init(&B.full[j], 1); tc::mbar_init(&B.empty[j], 2); }
    for (int j = 0; j < CT_NA; ++j) { tc::mbar_init(&B.afull[j], 1); tc::mbar_init(&B.aempty[j], 1); }
    for (int j = 0; j < 2; ++j) {
      tc::mbar_init(&B.sfull[j], 1);
      tc::mbar_init(&B.pfull[j], 4);
      tc::mbar_init(&B.pempty[j], 1);
      tc::mbar_init(&B.done[j], 1);
    }
    tc::mbar_init(B.sempty, 4);
    tc::mbar_init(B.tfull, 1);
    tc::mbar_init(B.tempty, 8);
    tc::mbar_init(B.never, 1);
    tc::mbar_fence_init();
    *abort_flag = 0;
  }
  for (int q = tid; q < CT_TQ; q += CT_THREADS) {
    const int i = i0 + q;
    int p = INT_MIN;
    if (i < Lq) {
      const int pp = q_pos ? q_pos[(size_t)b * Lq + i] : i;
      if (!is_mask_slot(pp)) p = pp;
    }
    posv[q] = p;
  }
  for (int c = tid; c < C; c += CT_THREADS) mask[c] = 0ull;
  __syncthreads();
  const int32_t* idx_t = idx + ((size_t)(b * Hkv + g) * Lq + i0) * K;
  auto entry_chunk = [&](int e) -> int {     // chunk of (row e / K, slot e % K), -1 if none
    const int q = e / K;
    if (posv[q] == INT_MIN) return -1;
    const int c = idx_t[e];
    if (c < 0) return -1;
    if (c >= C || !chunk_eligible(c, posv[q], w)) {
      if (flags & RDL_FLAG_CHECKS) record_status(RDL_ERR_DEVICE_CHECK);
      if (c >= C) return -1;
    }
    return c;
  };
  // bucket membership as row masks (a row selects a chunk at most once)
  const int nent = min(CT_TQ, Lq - i0) * K;
  for (int e = tid; e < nent; e += CT_THREADS) {
    const int c = entry_chunk(e);
    if (c >= 0) atomicOr(&mask[c], 1ull << (e / K));
  }
  __syncthreads();
  // exclusive scans of bucket sizes (entry offsets) and of non-empty flags (union slots):
  // per-thread runs of chunks, warp shuffles, then one warp over the warp totals
  {
    const int per = (C + CT_THREADS - 1) / CT_THREADS, c0 = tid * per, c1 = min(C, c0 + per);
    int l0 = 0, l1 = 0;
    for (int c = c0; c < c1; ++c) {
      const int n = __popcll(mask[c]);
      l0 += n;
      l1 += n > 0;
    }
    int s0 = l0, s1 = l1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int a0 = __shfl_up_sync(0xffffffffu, s0, off), a1 = __shfl_up_sync(0xffffffffu, s1, off);
      if (lane >= off) { s0 += a0; s1 += a1; }
    }
    if (lane == 31) { part[2 * warp] = s0; part[2 * warp + 1] = s1; }
    __syncthreads();
    if (warp == 0) {
      const int x0 = lane < CT_WARPS ? part[2 * lane] : 0, x1 = lane < CT_WARPS ? part[2 * lane + 1] : 0;
      int y0 = x0, y1 = x1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int a0 = __shfl_up_sync(0xffffffffu, y0, off), a1 = __shfl_up_sync(0xffffffffu, y1, off);
        if (lane >= off) { y0 += a0; y1 += a1; }
      }
      if (lane < CT_WARPS) { part[2 * lane] = y0 - x0; part[2 * lane + 1] = y1 - x1; }
      if (lane == 31) *nunion_s = y1;
    }
    __syncthreads();
    int r0 = part[2 * warp] + s0 - l0, r1 = part[2 * warp + 1] + s1 - l1;
    for (int c = c0; c < c1; ++c) {
      const int n = __popcll(mask[c]);
      ofs[c] = r0;
      if (n > 0) uni[r1++] = ct_union(c, r0, n);
      r0 += n;
    }
  }
  __syncthreads();
  // entries in ascending row order inside each bucket: rank = rows below q in the mask
  for (int e = tid; e < nent; e += CT_THREADS) {
    const int c = entry_chunk(e);
    if (c >= 0) {
      const int q = e / K;
      const int rank = __popcll(mask[c] & ((1ull << q) - 1ull));
      ent[ofs[c] + rank] = (uint16_t)((q << 8) | (e % K));
    }
  }
  // fixed partition per (row, head): M = max(window planes, z), Z = sum of exponentials
  const size_t plane_l = (size_t)gridDim.y / Hkv * Hq * Lq;
  for (int e = tid; e < CT_TQ * G; e += CT_THREADS) {
    const int q = e / G, h = e % G, i = i0 + q;
    if (posv[q] == INT_MIN) continue;
    const size_t li = (size_t)(b * Hq + g * G + h) * Lq + i;
    const float* zr = z_sel + li * K;
    float M = -INFINITY, Z = 0.f;
    if (K <= 32) {                              // all loads in flight at once
      float zz[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) zz[u] = u < K ? zr[u] : -INFINITY;
#pragma unroll
      for (int u = 0; u < 32; ++u) M = fmaxf(M, zz[u]);
      for (int sw = 0; sw < nsw; ++sw) M = fmaxf(M, lam_loc[sw * plane_l + li]);
      if (M == -INFINITY) M = 0.f;
#pragma unroll
      for (int u = 0; u < 32; ++u) Z += expf(zz[u] - M);
    } else {
      for (int s0 = 0; s0 < K; s0 += 8) {
        float zz[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) zz[u] = s0 + u < K ? zr[s0 + u] : -INFINITY;
#pragma unroll
        for (int u = 0; u < 8; ++u) M = fmaxf(M, zz[u]);
      }
      for (int sw = 0; sw < nsw; ++sw) M = fmaxf(M, lam_loc[sw * plane_l + li]);
      if (M == -INFINITY) M = 0.f;
      for (int s0 = 0; s0 < K; s0 += 8) {
        float zz[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) zz[u] = s0 + u < K ? zr[s0 + u] : -INFINITY;
#pragma unroll
        for (int u = 0; u < 8; ++u) Z += expf(zz[u] - M);
      }
    }
    float ls1 = -INFINITY;
    for (int sw = 0; sw < nsw; ++sw) {
      const float ls = lam_loc[sw * plane_l + li];
      if (ls != -INFINITY) Z += expf(ls - M);
      if (sw == 0) ls1 = ls;
    }
    Mw[q * 8 + h] = M;
    iZ[q * 8 + h] = Z > 0.f ? 1.f / Z : 0.f;
    // mass of the (single-plane) window part, used by the epilogue
    Ww[q * 8 + h] = (nsw == 1 && ls1 != -INFINITY && Z > 0.f) ? expf(ls1 - M) / Z : 0.f;
    if (lse) lse[li] = Z > 0.f ? M + logf(Z) : -INFINITY;
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_s;
  const int U = *nunion_s;
  // zero the home accumulators
  if (warp >= 11 && warp < 15) {
    const int qw = warp & 3;
    const float z8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int c0 = 0; c0 < CT_HOME; c0 += 8) tc::tmem_st8(tc::taddr(tbase, 32 * qw, c0), z8);
    tc::tmem_wait_st();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();

  const uint32_t smem_base = smem_u32(sm);
  // base descriptors (slot / buffer 0): Q rows and K are K-major, V^T is MN-major, P K-major.
  // The start-address field is the low 14 bits (address >> 4) and never carries inside the
  // shared window, so buffer / step offsets are added to these.
  const uint64_t dA0 = tc::sdesc(smem_base + CT_OFF_A, 16, 2048);
  const uint64_t dK0 = tc::sdesc(smem_base + CT_OFF_KV, 16, 1024);
  const uint64_t dV0 = tc::sdesc(smem_base + CT_OFF_KV + 16384, 8192, 1024);
  const uint64_t dP0 = tc::sdesc(smem_base + CT_OFF_P, 16, 1024);
  // passes: chunk u of the union, queries p0 .. p0+7 of its bucket; pass k uses Q buffer
  // k % NA and P buffer k & 1
  auto next_pass = [&](int& u, int& p0) {
    p0 += CT_QP;
    if (p0 >= (int)(uni[u] >> 24)) { ++u; p0 = 0; }
  };

  // ---------------------------------------------------------------- Q producer
  if (warp == 0) {
    if (lane == 0) {
      int k = 0;
      bool ok = true;
      for (int u = 0; u < U && ok; ++u) {
        const uint32_t un = uni[u];
        const int start = (un >> 12) & 4095, n = un >> 24;
        for (int p0 = 0; p0 < n; p0 += CT_QP, ++k) {
          const int nq = min(CT_QP, n - p0), ab = k % CT_NA;
          if (!ct_wait(&B.aempty[ab], ((k / CT_NA) & 1) ^ 1, abort_flag)) { ok = false; break; }
          unsigned char* at = sm + CT_OFF_A + ab * 16384;
          tc::mbar_arrive_expect_tx(&B.afull[ab], nq * 2048);
          // one box per run of consecutive query tokens (bucket rows ascend)
          for (int j = 0; j < nq;) {
            const int ql = ent[start + p0 + j] >> 8;
            int r = 1;
            while (j + r < nq && (ent[start + p0 + j + r] >> 8) == ql + r) ++r;
            tc::tma_load_4d(at + j * 2048, &maps.q[r - 1], 0, g * G, 0, b * Lq + i0 + ql, &B.afull[ab]);
            j += r;
          }
        }
      }
    }
  }
  // ---------------------------------------------------------------- K/V producer
  else if (warp == CT_KV_WARP) {
    if (lane == 0) {
      for (int u = 0; u < U; ++u) {
        const int c = uni[u] & 4095, slot = u % CT_NSLOT;
        if (!ct_wait(&B.empty[slot], ((u / CT_NSLOT) & 1) ^ 1, abort_flag)) break;
        unsigned char* kv = sm + CT_OFF_KV + slot * 32768;
        tc::mbar_arrive_expect_tx(&B.full[slot], 32768);
        const int krow = (b * Hkv + g) * L + c * S;
        tc::tma_load_3d(kv, &maps.k, 0, krow, 0, &B.full[slot]);
        tc::tma_load_3d(kv + 16384, &maps.v, 0, krow, 0, &B.full[slot]);
      }
    }
  }
  // ---------------------------------------------------------------- S MMAs
  // (the whole warp runs the issue loop; one elected lane issues: warp-uniform issue keeps
  // the descriptors in uniform registers)
  else if (warp == 1) {
    const uint32_t idesc_s = tc::idesc_bf16(64, 64, false, false);
    const uint32_t dS = tbase + (uint32_t)CT_SCOL;
    int k = 0;
    bool ok = true, issued = false;
    for (int u = 0; u < U && ok; ++u) {
      const int n = __shfl_sync(0xffffffffu, (int)(uni[u] >> 24), 0), slot = u % CT_NSLOT;
      if (!__all_sync(0xffffffffu, ct_wait(&B.full[slot], (u / CT_NSLOT) & 1, abort_flag))) break;
      if ((flags & RDL_FLAG_WAIT_TEST) && u == 0) {
        // a wait on a barrier nothing arrives on runs out: the failure path of every wait
        bool got = false;
        for (unsigned x = 0; x < CT_TEST_POLLS && !got; ++x) got = tc::mbar_try_wait(B.never, 0);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) {
            record_status(RDL_ERR_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
      }
      const uint64_t dk = dK0 + (uint64_t)((slot * 32768) >> 4);
      for (int p0 = 0; p0 < n; p0 += CT_QP, ++k) {
        const int ab = k % CT_NA, sb = k & 1;
        const bool w_ok = ct_wait(&B.afull[ab], (k / CT_NA) & 1, abort_flag) &&
                          ct_wait(B.sempty, (k & 1) ^ 1, abort_flag);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t da = dA0 + (uint64_t)((ab * 16384) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {      // K steps of 16: halves at +1 KB (Q) / +8 KB (K)
          const uint64_t qoff = (uint64_t)((ks >> 2) * 64 + (ks & 3) * 2);
          const uint64_t koff = (uint64_t)((ks >> 2) * 512 + (ks & 3) * 2);
          tc::mma_bf16_ss_warp(dS, da + qoff, dk + koff, idesc_s, ks > 0);
        }
        tc::mma_commit_warp(&B.sfull[sb]);
        tc::mma_commit_warp(&B.aempty[ab]);
        if (p0 + CT_QP >= n) tc::mma_commit_warp(&B.empty[slot]);     // K of this chunk done
        issued = true;
      }
    }
    if (issued) tc::mma_commit_warp(&B.done[0]); else tc::mbar_arrive_warp(&B.done[0]);
    tc::mbar_wait(&B.done[0], 0);          // bounded; not cut short by an abort
    __syncwarp();
  }
  // ---------------------------------------------------------------- PV MMAs
  else if (warp == 2) {
    const uint32_t dT = tbase + (uint32_t)CT_TCOL;
    int k = 0;
    bool ok = true, issued = false;
    for (int u = 0; u < U && ok; ++u) {
      const int n = __shfl_sync(0xffffffffu, (int)(uni[u] >> 24), 0), slot = u % CT_NSLOT;
      if (!__all_sync(0xffffffffu, ct_wait(&B.full[slot], (u / CT_NSLOT) & 1, abort_flag))) break;
      const uint64_t ad0 = dV0 + (uint64_t)((slot * 32768) >> 4);
      for (int p0 = 0; p0 < n; p0 += CT_QP, ++k) {
        const int nq = min(CT_QP, n - p0), pb = k & 1;
        const bool w_ok = ct_wait(&B.pfull[pb], (k >> 1) & 1, abort_flag) &&
                          ct_wait(B.tempty, (k & 1) ^ 1, abort_flag);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t bd0 = dP0 + (uint64_t)((pb * 8192) >> 4);
        // N rounded up to a multiple of 16; P rows past 8*nq are zero
        const uint32_t idesc_pv = tc::idesc_bf16(128, 16 * ((nq + 1) >> 1), true, false);
        tc::mma_bf16_ss_warp(dT, ad0, bd0, idesc_pv, false);
        tc::mma_bf16_ss_warp(dT, ad0 + 128, bd0 + 2, idesc_pv, true);
        tc::mma_bf16_ss_warp(dT, ad0 + 256, bd0 + 4, idesc_pv, true);
        tc::mma_bf16_ss_warp(dT, ad0 + 384, bd0 + 6, idesc_pv, true);
        tc::mma_commit_warp(B.tfull);
        tc::mma_commit_warp(&B.pempty[pb]);
        if (p0 + CT_QP >= n) tc::mma_commit_warp(&B.empty[slot]);     // V of this chunk done
        issued = true;
      }
    }
    if (issued) tc::mma_commit_warp(&B.done[1]); else tc::mbar_arrive_warp(&B.done[1]);
    tc::mbar_wait(&B.done[1], 0);
    __syncwarp();
  }
  // ---------------------------------------------------------------- softmax groups
  else if (warp <= 10) {
    const int grp = (warp - 3) >> 2;               // passes k with k % 2 == grp
    const int qw = warp & 3;                       // TMEM lane quarter of this warp
    const float sl2 = rsqrtf(128.f) * LOG2E;
    const int hh = lane >> 2, cq = 2 * (lane & 3);  // head row, column pair in each 8-group
    const int jqa = 2 * qw, jqb = 2 * qw + 1;       // queries of rows 16qw + hh and +8
    // per-row weight w = e^{z - M} / Z of a pass (raw z loaded one pass ahead)
    struct RowW { float za, ma, iza, zb, mb, izb; };
    auto pass_row = [&](int u, int p0) -> RowW {
      RowW r{-INFINITY, 0.f, 0.f, -INFINITY, 0.f, 0.f};
      if (u >= U || hh >= G) return r;
      const uint32_t un = uni[u];
      const int start = (un >> 12) & 4095, nq = min(CT_QP, (int)(un >> 24) - p0);
      const float* zh = z_sel + ((size_t)(b * Hq + g * G + hh) * Lq + i0) * K;
      if (jqa < nq) {
        const uint16_t en = ent[start + p0 + jqa];
        r.za = zh[(size_t)(en >> 8) * K + (en & 255)];
        r.ma = Mw[(en >> 8) * 8 + hh];
        r.iza = iZ[(en >> 8) * 8 + hh];
      }
      if (jqb < nq) {
        const uint16_t en = ent[start + p0 + jqb];
        r.zb = zh[(size_t)(en >> 8) * K + (en & 255)];
        r.mb = Mw[(en >> 8) * 8 + hh];
        r.izb = iZ[(en >> 8) * 8 + hh];
      }
      return r;
    };
    int u = 0, p0 = 0;
    if (grp == 1 && U > 0) next_pass(u, p0);
    RowW wnext = pass_row(u, p0);
    for (int m = 0; u < U; ++m) {
      const int nq = min(CT_QP, (int)(uni[u] >> 24) - p0);
      const RowW wc = wnext;
      next_pass(u, p0);
      if (u < U) next_pass(u, p0);                 // this group's next pass
      wnext = pass_row(u, p0);
      if (!ct_wait(&B.sfull[grp], m & 1, abort_flag)) break;
      tc::tc_fence_after();
      float sv[32];
      tc::tmem_ld16x256b_x8(tc::taddr(tbase, 32 * qw, CT_SCOL), sv);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(B.sempty);    // S region free for the next pass
      const bool va = jqa < nq && hh < G, vb = jqb < nq && hh < G;
      // sv[4i + 0,1]: row a, columns 8i + cq + {0,1}; sv[4i + 2,3]: row b, same columns.
      // Column 63 (the routing-mask slot) is i = 7, cq = 6, second element.
      const bool last = cq == 6;
      float ma = fmaxf(sv[0], sv[1]), mb = fmaxf(sv[2], sv[3]);
#pragma unroll
      for (int i = 1; i < 8; ++i) {
        ma = fmaxf(ma, (i == 7 && last) ? sv[4 * i] : fmaxf(sv[4 * i], sv[4 * i + 1]));
        mb = fmaxf(mb, (i == 7 && last) ? sv[4 * i + 2] : fmaxf(sv[4 * i + 2], sv[4 * i + 3]));
      }
      ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 1));
      mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
      ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 2));
      mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
      const float oa = va ? ma * sl2 : 0.f, ob = vb ? mb * sl2 : 0.f;
      float la0 = 0.f, la1 = 0.f, lb0 = 0.f, lb1 = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool mask1 = i == 7 && last;
        sv[4 * i] = fast_exp2(fmaf(sv[4 * i], sl2, -oa));
        sv[4 * i + 1] = mask1 ? 0.f : fast_exp2(fmaf(sv[4 * i + 1], sl2, -oa));
        sv[4 * i + 2] = fast_exp2(fmaf(sv[4 * i + 2], sl2, -ob));
        sv[4 * i + 3] = mask1 ? 0.f : fast_exp2(fmaf(sv[4 * i + 3], sl2, -ob));
        la0 += sv[4 * i];
        la1 += sv[4 * i + 1];
        lb0 += sv[4 * i + 2];
        lb1 += sv[4 * i + 3];
      }
      float la = la0 + la1, lb = lb0 + lb1;
      la += __shfl_xor_sync(0xffffffffu, la, 1);
      lb += __shfl_xor_sync(0xffffffffu, lb, 1);
      la += __shfl_xor_sync(0xffffffffu, la, 2);
      lb += __shfl_xor_sync(0xffffffffu, lb, 2);
      const float fa = (va && la > 0.f) ? expf(wc.za - wc.ma) * wc.iza / la : 0.f;
      const float fb = (vb && lb > 0.f) ? expf(wc.zb - wc.mb) * wc.izb / lb : 0.f;
      if (!ct_wait(&B.pempty[grp], (m & 1) ^ 1, abort_flag)) break;
      unsigned char* pt = sm + CT_OFF_P + grp * 8192;
      const int ra = 16 * qw + hh, rb = ra + 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t wa = va ? pack_bf16(sv[4 * i] * fa, sv[4 * i + 1] * fa) : 0u;
        const uint32_t wb = vb ? pack_bf16(sv[4 * i + 2] * fb, sv[4 * i + 3] * fb) : 0u;
        *reinterpret_cast<uint32_t*>(pt + tc::sw128(ra, 8 * i + cq)) = wa;
        *reinterpret_cast<uint32_t*>(pt + tc::sw128(rb, 8 * i + cq)) = wb;
      }
      tc::fence_proxy_async();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&B.pfull[grp]);
    }
  }
  // ---------------------------------------------------------------- home adds
  else if (warp <= 18) {
    const int qw = warp & 3;
    const int hs = 4 * ((warp - 11) >> 2);         // heads hs .. hs+3 of every query
    const uint32_t lanebase = tc::taddr(tbase, 32 * qw, 0);
    int k = 0;
    bool ok = true;
    for (int u = 0; u < U && ok; ++u) {
      const uint32_t un = uni[u];
      const int start = (un >> 12) & 4095, n = un >> 24;
      for (int p0 = 0; p0 < n && ok; p0 += CT_QP, ++k) {
        const int nq = min(CT_QP, n - p0);
        // home column of query j of this pass, held by lane j
        const int hcol = lane < nq ? (ent[start + p0 + lane] >> 8) * CT_HP + hs : 0;
        if (!ct_wait(B.tfull, k & 1, abort_flag)) { ok = false; break; }
        tc::tc_fence_after();
        if (hs < G) {
          for (int j0 = 0; j0 < nq; j0 += 4) {      // 4 queries per round trip
            float t4[4][4], h4[4][4];
            int hc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              hc[j] = __shfl_sync(0xffffffffu, hcol, (j0 + j) & 31);
              if (j0 + j < nq) {
                tc::tmem_ld4(lanebase + (uint32_t)(CT_TCOL + 8 * (j0 + j) + hs), t4[j]);
                tc::tmem_ld4(lanebase + (uint32_t)hc[j], h4[j]);
              }
            }
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if (j0 + j < nq) {
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) h4[j][e2] += t4[j][e2];
                tc::tmem_st4(lanebase + (uint32_t)hc[j], h4[j]);
              }
            }
          }
          tc::tmem_wait_st();
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(B.tempty);
      }
    }
  }
  // ---------------------------------------------------------------- epilogue
  // home columns + window part -> o; warps 3-18, four per TMEM lane quarter, take every
  // fourth query (each warp writes its 32 head-dim lanes)
  if (warp >= 3 && warp <= 18) {
    ct_epi_sync();
    if (!*abort_flag) {
      tc::tc_fence_after();
      const int qw = warp & 3, e4 = (warp - 3) >> 2;
      const int d = 32 * qw + lane;
      const size_t plane = (size_t)gridDim.y / Hkv * Lq * Hq * 128;
      const int qn = min(CT_TQ, Lq - i0);
      auto load_ol = [&](int q, float* ol) {
        const bool on = nsw == 1 && q < qn && posv[q] != INT_MIN;
        const float* olr = o_loc + ((size_t)(b * Lq + i0 + q) * Hq + g * G) * 128 + d;
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) ol[e2] = (on && e2 < G) ? olr[e2 * 128] : 0.f;
      };
      float ol0[8], ol1[8], ol2[8];                // window rows of queries q, q+4, q+8
      load_ol(e4, ol0);
      load_ol(e4 + 4, ol1);
      for (int q = e4; q < qn; q += 4) {
        load_ol(q + 8, ol2);
        float acc[8];
        tc::tmem_ld8(tc::taddr(tbase, 32 * qw, q * CT_HP), acc);
        tc::tmem_wait_ld();
        if (posv[q] != INT_MIN) {
          const int i = i0 + q;
          __nv_bfloat16* orow = o + ((size_t)(b * Lq + i) * Hq + g * G) * 128;
          if (nsw == 1) {
#pragma unroll
            for (int e2 = 0; e2 < 8; ++e2)
              if (e2 < G) orow[e2 * 128 + d] = __float2bfloat16_rn(acc[e2] + Ww[q * 8 + e2] * ol0[e2]);
          } else {
            const float* olr = o_loc + ((size_t)(b * Lq + i) * Hq + g * G) * 128 + d;
            for (int e2 = 0; e2 < G; ++e2) {
              const size_t li = (size_t)(b * Hq + g * G + e2) * Lq + i;
              float v = acc[e2];
              for (int sw = 0; sw < nsw; ++sw) {
                const float ls = lam_loc[sw * plane_l + li];
                if (ls != -INFINITY) v += expf(ls - Mw[q * 8 + e2]) * iZ[q * 8 + e2] * olr[sw * plane + e2 * 128];
              }
              orow[e2 * 128 + d] = __float2bfloat16_rn(v);
            }
          }
        }
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) { ol0[e2] = ol1[e2]; ol1[e2] = ol2[e2]; }
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

}  // namespace rdl
