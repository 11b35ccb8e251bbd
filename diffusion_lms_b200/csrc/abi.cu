// C ABI of librdl.so (declared in include/rdl.h): argument checks on the host, workspace
// layout and kernel dispatch.  Nothing here allocates, frees or synchronises (apart from
// rdl_last_device_status, which is documented to synchronise).
#include <atomic>
#include <mutex>
#include <type_traits>
#include <climits>
#include <cstdint>
#include <cstdio>

#include "common.cuh"
#include "summary_pool.cuh"
#include "score.cuh"
#include "score_mma.cuh"
#include "decode_score.cuh"
#include "window_attn.cuh"
#include "chunk_attn.cuh"
#include "tmap.cuh"
#include "chunk_tc.cuh"
#include "chunk_major.cuh"
#include "window_tc.cuh"
#include "score_tc.cuh"
#include "decode.cuh"
#include <cstdlib>

using namespace rdl;

namespace rdl {
static std::atomic<unsigned long long> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }
}  // namespace rdl

namespace {

constexpr int kMaxK = 64;
constexpr int kMaxR = 128;
constexpr int kMaxC = 8192;        // top-K keeps a whole score row per warp in shared memory

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bool dims_ok(const rdl_dims* dm) {
  if (!dm) return false;
  if (dm->B < 1 || dm->L < S || dm->L % S != 0 || dm->Lq < 1) return false;
  if (dm->Hq < 1 || dm->Hkv < 1 || dm->Hq % dm->Hkv != 0) return false;
  if (dm->d != 64 && dm->d != 128) return false;
  const long long rows = (long long)dm->B * dm->Lq * dm->Hq * dm->d;
  const long long kv = (long long)dm->B * dm->Hkv * dm->L * dm->d;
  if (rows > (1LL << 40) || kv > (1LL << 40)) return false;
  return true;
}
bool dtype_ok(rdl_dtype t) { return t == RDL_BF16 || t == RDL_F32; }
bool route_dims_ok(const rdl_dims* dm) {
  if (!dims_ok(dm)) return false;
  const int C = dm->L / S;
  if (dm->K < 1 || dm->K > kMaxK || dm->K > C) return false;
  if (dm->r < 0 || dm->r > kMaxR) return false;
  if (dm->r > 0 && dm->D < 1) return false;
  return true;
}
// bf16, head dim 128 and at most 8 heads per group run on the tensor-core kernels;
// everything else on the scalar kernels.
bool fast_attn(const rdl_dims* dm, rdl_dtype t) {
  return t == RDL_BF16 && dm->d == 128 && dm->Hq / dm->Hkv <= 8;
}
// Chunk splits of the selected-chunk pass when there are few (row, group) items.
int attn_splits(const rdl_dims* dm) {
  const long long items = (long long)dm->B * dm->Lq * dm->Hkv;
  if (items >= 4096) return 1;
  int ns = (int)((4096 + items - 1) / items);
  if (ns > 16) ns = 16;
  return ns < dm->K ? ns : dm->K;
}
// Key splits of the window pass when there are few 16-row tiles (decode blocks).
int window_splits(const rdl_dims* dm) {
  if (dm->w < 0) return 1;
  const long long ctas = (long long)dm->B * ((dm->Lq + WIN_ROWS - 1) / WIN_ROWS) * dm->Hkv;
  if (ctas >= 148) return 1;
  const long long want = (296 + ctas - 1) / ctas;
  const long long blocks = (2LL * dm->w + WIN_ROWS + WIN_KEYS - 1) / WIN_KEYS + 1;
  long long ns = want < blocks ? want : blocks;
  return ns < 1 ? 1 : (int)ns;
}

// The tensor-core score path: bf16, d = 128, rank 64 residual with D % 64 == 0, and
// enough query rows to fill 128-row tiles.  Everything else runs the fp32 path.
constexpr int kFastScoreMinRows = 128;
bool fast_score(const rdl_dims* dm, rdl_dtype t) {
  return t == RDL_BF16 && dm->d == 128 && dm->r == 64 && dm->D % 64 == 0 && dm->Hq / dm->Hkv <= 8 &&
         dm->Lq >= kFastScoreMinRows;
}
// The tensor-core scorer in two passes around the top-K, without a per-head score buffer, once
// that buffer would pass 1 GiB (long sequences); below, one pass writing every per-head score.
bool fused_score(const rdl_dims* dm, rdl_dtype t) {
  return fast_score(dm, t) && sizeof(float) * (size_t)dm->B * dm->Hq * dm->Lq * (dm->L / S) > (size_t(1) << 30);
}
// decode blocks: few rows, head dim 128 -> the decode score path
bool decode_score_path(const rdl_dims* dm) { return dm->d == 128 && dm->Lq <= 64; }

// Decode blocks on the chained kernels of decode.cuh: bf16, head dim 128, at most 64 rows
// per sequence, at most 8 heads per group, residual rank 0, 64 or 128.
constexpr int kSMs = 148;
bool dec_rows_ok(const rdl_dims* dm, rdl_dtype t) {
  return t == RDL_BF16 && dm->d == 128 && dm->Lq <= 64 && dm->Hq / dm->Hkv <= 8;
}
bool dec_score_ok(const rdl_dims* dm, rdl_dtype t) {
  return dec_rows_ok(dm, t) && dm->K <= kMaxK &&
         (dm->r == 0 || ((dm->r == 64 || dm->r == 128) && dm->D % 64 == 0));
}
// decode attention (chunk-major, balanced): at most 32 rows and 2048 chunks per sequence,
// at most 64 window slabs per row
bool dec_attn_rows_ok(const rdl_dims* dm, rdl_dtype t) {
  return t == RDL_BF16 && dm->d == 128 && dm->Lq <= dec::AT_QROWS && dm->Hq / dm->Hkv <= 8 &&
         dm->L / S <= dec::AT_MAXC && dec::max_win_slabs(dm->w) <= 64;
}
bool dec_attn_ok(const rdl_dims* dm, rdl_dtype t) { return dec_attn_rows_ok(dm, t) && dm->K <= kMaxK; }
bool dec_swa_ok(const rdl_dims* dm, rdl_dtype t) { return dec_attn_rows_ok(dm, t) && dm->w >= 0; }
int dec_attn_stages(const rdl_dims* dm, int K) {
  for (int st = 4; st >= 2; --st)
    if (dec::attn_smem(st, dm->Lq, K, dm->L / S).total <= 232448) return st;
  return 0;
}
int dec_attn_ranges(const rdl_dims* dm) {
  const int r = kSMs / (dm->B * dm->Hkv);
  return r < 1 ? 1 : r;
}
// score grid: (ranges, Hq, B); each range streams boxes of SC_BOXR summary rows through a
// ring as deep as shared memory allows (loaded before the dependency wait)
struct DecScoreGrid {
  int MT, ranges, ncr, nstg, smem;
};
DecScoreGrid dec_score_grid(const rdl_dims* dm) {
  DecScoreGrid gr{};
  const int C = dm->L / S;
  gr.MT = dm->Lq <= 16 ? 1 : (dm->Lq <= 32 ? 2 : 4);
  int ranges = kSMs / (dm->B * dm->Hq);
  if (ranges < 1) ranges = 1;
  int ncr = (C + ranges - 1) / ranges;
  ncr = (ncr + 7) & ~7;
  gr.ranges = (C + ncr - 1) / ncr;
  gr.ncr = ncr;
  const int nbox = (ncr + dec::SC_BOXR - 1) / dec::SC_BOXR;
  gr.nstg = 0;
  for (int nstg = 4; nstg >= 1; --nstg)
    if (dec::score_smem(gr.MT, dm->r, nstg, ncr).total <= 232448) {
      gr.nstg = nstg < nbox ? nstg : nbox;
      break;
    }
  gr.smem = gr.nstg > 0 ? dec::score_smem(gr.MT, dm->r, gr.nstg, ncr).total : 0;
  return gr;
}
bool use_pdl() {
  static const bool on = [] {
    const char* e = std::getenv("RDL_NO_PDL");
    return !(e && e[0] == '1');
  }();
  return on;
}
// Launch with programmatic dependent launch allowed (the kernel waits on its predecessor
// with griddepcontrol.wait before touching anything the predecessor may write).
template <typename... Exp, typename... Act>
cudaError_t launch_ex(bool pdl, void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      Act&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = (pdl && use_pdl()) ? 1 : 0;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
}
template <typename... Exp, typename... Act>
cudaError_t launch_pdl(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Act&&... args) {
  return launch_ex(true, kern, grid, block, smem, st, std::forward<Act>(args)...);
}
struct ScoreWs {
  size_t t, qres, z_all, zeta, tt, sb, tpart, total;
};
ScoreWs score_ws(const rdl_dims* dm, rdl_dtype dt) {
  const size_t C = dm->L / S;
  ScoreWs w{};
  size_t off = 0;
  if (fused_score(dm, dt)) {
    // the group maxima, the split residual rows and the split summary rows (no per-head scores)
    w.zeta = off; off += align256(sizeof(float) * (size_t)dm->B * dm->Hkv * dm->Lq * C);
    w.tt = off;  off += align256(sizeof(__nv_bfloat16) * (size_t)dm->B * dm->Lq * 2 * dm->r);
    w.sb = off;  off += align256(sizeof(__nv_bfloat16) * (size_t)dm->B * dm->Hq * C * (2 * dm->d + 2 * dm->r));
    w.total = off;
    return w;
  }
  w.z_all = off; off += align256(sizeof(float) * (size_t)dm->B * dm->Hq * dm->Lq * C);
  w.zeta = off;
  if (dec_score_ok(dm, dt)) {
    // the hidden-slice partials of t, summed by the scorer
    w.t = off;     off += align256(sizeof(float) * dec::TK_CL * (size_t)dm->B * dm->Lq * (dm->r > 0 ? dm->r : 1));
  } else {
    off += align256(sizeof(float) * (size_t)dm->B * dm->Hkv * dm->Lq * C);
  }
  if (dec_score_ok(dm, dt)) {
  } else if (fast_score(dm, dt)) {
    w.tt = off;  off += align256(sizeof(__nv_bfloat16) * (size_t)dm->B * dm->Lq * 2 * dm->r);
    w.sb = off;  off += align256(sizeof(__nv_bfloat16) * (size_t)dm->B * dm->Hq * C * (2 * dm->d + 2 * dm->r));
  } else {
    w.t = off;     off += align256(sizeof(float) * (size_t)dm->B * dm->Lq * (dm->r > 0 ? dm->r : 1));
    w.qres = off;  off += align256(sizeof(float) * (size_t)dm->B * dm->Lq * dm->Hq * dm->d);
    if (decode_score_path(dm) && dm->r > 0) {
      const size_t nsl = (dm->D + DQ_KS - 1) / DQ_KS;
      w.tpart = off; off += align256(sizeof(float) * nsl * dm->B * dm->Lq * dm->r);
    }
  }
  w.total = off;
  return w;
}
struct AttnWs {
  size_t o_loc, lam_loc, o_acc, total;
  size_t zero, zero_bytes, counts, cursor, nitems, offs, list, items, part;   // chunk-major path
};
// Prefill route attention chunk-major over the whole sequence (chunk_major.cuh): fast shapes
// whose selections fit the entry encoding (row << 6 | slot).
bool cm_path_ok(const rdl_dims* dm, rdl_dtype t) {
  return fast_attn(dm, t) && dm->L / S <= CM_MAXC && dm->K <= 64 && dm->Lq < (1 << 25);
}
// The row-tile kernel (chunk_tc.cuh) shares each chunk's K/V among the rows of a 45-row tile that
// selected it; when those buckets average fewer than 4 rows (long sequences: about 45 K / C)
// the chunk-major path, which gathers every row of a chunk, takes over.
bool use_chunk_major(const rdl_dims* dm, rdl_dtype t) {
  return cm_path_ok(dm, t) && (double)CT_TQ * dm->K < 4.0 * (dm->L / S);
}
size_t cm_max_items(const rdl_dims* dm) {
  const size_t bg = (size_t)dm->B * dm->Hkv, C = dm->L / S;
  return (bg * dm->Lq * dm->K + CM_IT - 1) / CM_IT + bg * C;
}
AttnWs attn_ws(const rdl_dims* dm, rdl_dtype t) {
  AttnWs w{};
  if (!fast_attn(dm, t)) return w;
  if (dec_attn_ok(dm, t) && dec_attn_stages(dm, dm->K) > 0) {
    // chunk outputs [B, Lq, Hkv, K, G, d], the window part's unnormalised vector
    // [B, Lq, Hq, d] and its (max, sum) [B, Lq, Hq]
    const size_t rows = (size_t)dm->B * dm->Lq * dm->Hq;
    size_t off = 0;
    w.o_acc = off;   off += align256(sizeof(float) * rows * dm->K * dm->d);
    w.o_loc = off;   off += align256(sizeof(float) * rows * dm->d);
    w.lam_loc = off; off += align256(sizeof(float2) * rows);
    w.total = off;
    return w;
  }
  const size_t rows = (size_t)dm->B * dm->Lq * dm->Hq;
  size_t off = 0;
  const int nsw = window_splits(dm);
  w.o_loc = off;   off += align256(sizeof(float) * rows * dm->d * nsw);
  w.lam_loc = off; off += align256(sizeof(float) * rows * nsw);
  w.o_acc = off;
  if (use_chunk_major(dm, t)) {
    // bucket counts, cursors and the item count (zeroed by one memset), bucket offsets, the
    // bucketed selections, the work items and the fp16 chunk outputs [B*Hkv, Lq, K, G, d]
    const size_t bg = (size_t)dm->B * dm->Hkv, C = dm->L / S, G = dm->Hq / dm->Hkv;
    w.zero = off;
    w.counts = off;  off += sizeof(int) * bg * C;
    w.cursor = off;  off += sizeof(int) * bg * C;
    w.nitems = off;  off += sizeof(int);
    w.zero_bytes = off - w.zero;
    off = align256(off);
    w.offs = off;    off += align256(sizeof(int) * bg * C);
    w.list = off;    off += align256(sizeof(int) * bg * dm->Lq * dm->K);
    w.items = off;   off += align256(sizeof(CmItem) * cm_max_items(dm));
    w.part = off;    off += align256(sizeof(__half) * bg * dm->Lq * dm->K * G * dm->d);
    w.total = off;
    return w;
  }
  const int ns = attn_splits(dm);
  if (ns > 1) off += align256(sizeof(float) * rows * dm->d * ns);
  w.total = off;
  return w;
}

rdl_status attn_chunk_major(const void* q, const int32_t* q_pos, const void* k, const void* v, const int32_t* idx,
                            const float* z_sel, const rdl_dims* dm, void* o, float* lse, void* workspace,
                            cudaStream_t st);

// Sliding-window workspace: key-split partials when the row count is small (else none).
size_t swa_ws(const rdl_dims* dm, rdl_dtype t) {
  if (!fast_attn(dm, t) || dm->w < 0) return 0;
  if (dec_swa_ok(dm, t)) return 0;
  const int nsw = window_splits(dm);
  if (nsw <= 1) return 0;
  const size_t rows = (size_t)dm->B * dm->Lq * dm->Hq;
  return align256(sizeof(float) * rows * dm->d * nsw) + align256(sizeof(float) * rows * nsw);
}

rdl_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RDL_OK : RDL_ERR_CUDA; }

// |p - j| <= w with p, j in [0, L) never exceeds L - 1, so a radius >= L means "everything"
// and any negative radius means "no window"; clamping keeps device index math in range.
rdl_dims clamp_w(const rdl_dims* d) {
  rdl_dims c = *d;
  if (c.w > c.L) c.w = c.L;
  if (c.w < 0) c.w = -1;
  return c;
}

rdl_status launch_topk(const float* zeta, const float* z_all, const int32_t* q_pos, const rdl_dims* dm,
                       int32_t* idx, float* z_sel, cudaStream_t st) {
  const int C = dm->L / S;
  if ((long long)dm->B * dm->Lq * dm->Hkv <= 1024) {
    // few rows: a CTA per (row, group)
    const size_t smem = (size_t)C * sizeof(uint32_t);
    if (cudaFuncSetAttribute(topk_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return RDL_ERR_CUDA;
    count_launch();
    topk_cta_kernel<<<dim3(dm->Lq * dm->Hkv, dm->B), 256, smem, st>>>(zeta, z_all, q_pos, dm->Lq, dm->L, dm->Hq,
                                                                      dm->Hkv, dm->K, idx, z_sel);
    return cuda_status(cudaGetLastError());
  }
  const int warps = 4;
  const size_t smem = (size_t)warps * topk_warp_words(C) * sizeof(uint32_t);
  if (cudaFuncSetAttribute(topk_radix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return RDL_ERR_CUDA;
  dim3 g4((unsigned)(((long long)dm->Lq * dm->Hkv + warps - 1) / warps), dm->B);
  count_launch();
  topk_radix_kernel<<<g4, warps * 32, smem, st>>>(zeta, z_all, q_pos, dm->Lq, dm->L, dm->Hq, dm->Hkv, dm->K,
                                                  idx, z_sel);
  return cuda_status(cudaGetLastError());
}

rdl_status score_decode(const void* q, const int32_t* q_pos, const void* x, const void* w_down,
                        const void* w_up, const float* summary, const float* entropy, const rdl_dims* dm,
                        int32_t* idx, float* z_sel, void* workspace, cudaStream_t st) {
  const ScoreWs wl = score_ws(dm, RDL_BF16);
  char* ws = static_cast<char*>(workspace);
  float* t = reinterpret_cast<float*>(ws + wl.t);
  float* z_all = reinterpret_cast<float*>(ws + wl.z_all);
  const int C = dm->L / S, M = dm->B * dm->Lq;
  const bool res = dm->r > 0 && x;
  const DecScoreGrid gr = dec_score_grid(dm);
  const bool split = (dm->flags & RDL_FLAG_SPLIT_SUMMARY) != 0;
  CUtensorMap smap;
  const unsigned long long srows = (unsigned long long)dm->B * dm->Hq * C;
  if (gr.nstg < 1) return RDL_ERR_UNSUPPORTED;
  if (split ? !make_tmap_split_rows(&smap, summary, srows, (unsigned)dec::SC_BOXR)
            : !make_tmap_f32_rows(&smap, summary, srows, (unsigned)dec::SC_BOXR))
    return RDL_ERR_CUDA;
  if (res) {
    const int slice = ((dm->D + dec::TK_CL * 64 - 1) / (dec::TK_CL * 64)) * 64;
    const int kc = slice < dec::TK_KMAX ? slice : dec::TK_KMAX;
    const int rows = ((M + 15) / 16) * 16;
    const int tsm = dec::tk_smem(rows, dm->r, kc);
    CUtensorMap xmap, wmap;
    if (!make_tmap_bf16(&xmap, x, (unsigned long long)M, (unsigned)dm->D, 64, (unsigned)rows) ||
        !make_tmap_bf16(&wmap, w_down, (unsigned long long)dm->D, (unsigned)dm->r, 64, 64))
      return RDL_ERR_CUDA;
    if (cudaFuncSetAttribute(dec::dec_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tsm) != cudaSuccess)
      return RDL_ERR_CUDA;
    if (launch_pdl(dec::dec_t_kernel, dim3(dec::TK_CL), dim3(256), tsm, st, xmap, wmap, M, dm->D, dm->r, kc, t) !=
        cudaSuccess)
      return RDL_ERR_CUDA;
  }
  auto kern = split ? (gr.MT == 1 ? dec::dec_score_kernel<1, true>
                                  : (gr.MT == 2 ? dec::dec_score_kernel<2, true> : dec::dec_score_kernel<4, true>))
                    : (gr.MT == 1 ? dec::dec_score_kernel<1, false>
                                  : (gr.MT == 2 ? dec::dec_score_kernel<2, false> : dec::dec_score_kernel<4, false>));
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, gr.smem) != cudaSuccess)
    return RDL_ERR_CUDA;
  const float tau = (float)(1.0 / sqrt((double)dm->d));
  // launched early only behind dec_t_kernel: its prologue loads inputs before the wait
  if (launch_ex(res, kern, dim3(gr.ranges, dm->Hq, dm->B), dim3(dec::SC_WARPS * 32), gr.smem, st, smap, summary,
                 static_cast<const __nv_bfloat16*>(q), q_pos, (const float*)(res ? t : nullptr),
                 static_cast<const __nv_bfloat16*>(w_up), entropy, dm->Lq, dm->L, dm->Hq, res ? dm->r : 0, dm->w, tau,
                 dm->lambda, gr.ncr, gr.nstg, z_all) != cudaSuccess)
    return RDL_ERR_CUDA;
  const int G = dm->Hq / dm->Hkv;
  const bool zs = C % 4 == 0 && G * C <= dec::DK_MAXZ;
  const size_t ksm = (size_t)(((C + 3) & ~3) + (zs ? G * C : 0)) * sizeof(uint32_t);
  auto tk = C <= 1024 ? (zs ? dec::dec_topk_kernel<true, 2> : dec::dec_topk_kernel<false, 2>)
            : C <= 2048 ? (zs ? dec::dec_topk_kernel<true, 4> : dec::dec_topk_kernel<false, 4>)
                        : (zs ? dec::dec_topk_kernel<true, 16> : dec::dec_topk_kernel<false, 16>);
  if (cudaFuncSetAttribute(tk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ksm) != cudaSuccess)
    return RDL_ERR_CUDA;
  if (launch_pdl(tk, dim3(dm->Lq, dm->Hkv, dm->B), dim3(dec::DK_THREADS), ksm, st, (const float*)z_all, q_pos, dm->Lq, dm->L,
                 dm->Hq, dm->Hkv, dm->K, idx, z_sel) != cudaSuccess)
    return RDL_ERR_CUDA;
  return RDL_OK;
}

rdl_status attn_decode(const void* q, const int32_t* q_pos, const void* k, const void* v, const int32_t* idx,
                       const float* z_sel, const rdl_dims* dm, void* o, float* lse, void* workspace,
                       cudaStream_t st) {
  const AttnWs wl = attn_ws(dm, RDL_BF16);
  char* ws = static_cast<char*>(workspace);
  float* o_part = reinterpret_cast<float*>(ws + wl.o_acc);
  float* ow = reinterpret_cast<float*>(ws + wl.o_loc);
  float2* ml = reinterpret_cast<float2*>(ws + wl.lam_loc);
  const unsigned long long kvrows = (unsigned long long)dm->B * dm->Hkv * dm->L;
  CUtensorMap kmap, vmap;
  if (!make_tmap_kv_halves(&kmap, k, kvrows) || !make_tmap_kv_halves(&vmap, v, kvrows)) return RDL_ERR_CUDA;
  const int stages = dec_attn_stages(dm, dm->K);
  const int smem = dec::attn_smem(stages, dm->Lq, dm->K, dm->L / S).total;
  const float sl2w = (float)(1.0 / sqrt((double)dm->d) * 1.4426950408889634);
  if (dm->w >= 0) {
    // the local window, while the top-K of the step may still run (reads inputs only)
    const int wsm = dec::swa_smem();
    if (cudaFuncSetAttribute(dec::dec_swa_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, wsm) !=
        cudaSuccess)
      return RDL_ERR_CUDA;
    const int ctas = dm->B * dm->Hkv * ((dm->Lq + 1) / 2);
    if (launch_pdl(dec::dec_swa_kernel<true>, dim3(ctas), dim3(dec::SW_WARPS * 32), wsm, st, kmap, vmap,
                   static_cast<const __nv_bfloat16*>(q), q_pos, dm->L, dm->Lq, dm->Hq, dm->Hkv, dm->w, sl2w,
                   (__nv_bfloat16*)nullptr, (float*)nullptr, ow, ml) != cudaSuccess)
      return RDL_ERR_CUDA;
  }
  auto kern = dec::dec_attn_kernel<true>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return RDL_ERR_CUDA;
  const float sl2 = (float)(1.0 / sqrt((double)dm->d) * 1.4426950408889634);
  const int R = dec_attn_ranges(dm);
  if (launch_pdl(kern, dim3(dm->B * dm->Hkv * R), dim3(dec::AT_THREADS), smem, st, kmap, vmap,
                 static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                 static_cast<const __nv_bfloat16*>(q), q_pos, idx, dm->L, dm->Lq, dm->Hq, dm->Hkv, dm->K, dm->w,
                 dm->flags, R, stages, sl2, o_part) != cudaSuccess)
    return RDL_ERR_CUDA;
  const long long items = (long long)dm->B * dm->Lq * dm->Hq;
  // The combine is launched early; its shared-memory request keeps it at one CTA per SM, so
  // its CTAs spread over the SMs as the attention CTAs retire instead of piling onto the
  // first free ones (measured 6 CTAs per SM and twice the time otherwise).
  if (cudaFuncSetAttribute(dec::dec_comb_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           dec::COMB_SPREAD_SMEM) != cudaSuccess)
    return RDL_ERR_CUDA;
  if (launch_pdl(dec::dec_comb_kernel<true>, dim3((unsigned)((items + 7) / 8)), dim3(256), dec::COMB_SPREAD_SMEM, st,
                 q_pos, idx, z_sel,
                 (const float*)o_part, (const float*)ow, (const float2*)ml, dm->B, dm->L, dm->Lq, dm->Hq,
                 dm->Hkv, dm->K, dm->w, dm->flags, static_cast<__nv_bfloat16*>(o), lse) != cudaSuccess)
    return RDL_ERR_CUDA;
  return RDL_OK;
}

rdl_status score_fast(const void* q, const int32_t* q_pos, const void* x, const void* w_down,
                      const void* w_up, const float* summary, const float* entropy,
                      const rdl_dims* dm, int32_t* idx, float* z_sel, void* workspace,
                      cudaStream_t st) {
  constexpr int R = 64;
  const ScoreWs wl = score_ws(dm, RDL_BF16);
  char* ws = static_cast<char*>(workspace);
  float* z_all = reinterpret_cast<float*>(ws + wl.z_all);
  float* zeta = reinterpret_cast<float*>(ws + wl.zeta);
  __nv_bfloat16* tt = reinterpret_cast<__nv_bfloat16*>(ws + wl.tt);
  __nv_bfloat16* sb = reinterpret_cast<__nv_bfloat16*>(ws + wl.sb);
  const int M = dm->B * dm->Lq, C = dm->L / S;
  {
    auto kern = xw_mma_kernel<R>;
    const int smem = 2 * XW_ROWS * 128 + 2 * XW_KB * R * 2;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return RDL_ERR_CUDA;
    count_launch();
    kern<<<(M + XW_ROWS - 1) / XW_ROWS, 128, smem, st>>>(static_cast<const __nv_bfloat16*>(x),
                                                         static_cast<const __nv_bfloat16*>(w_down), M, dm->D, tt);
  }
  {
    const int smem = (R * 129 + 8 * 128) * (int)sizeof(float);
    auto kern = sprep_kernel<R>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return RDL_ERR_CUDA;
    count_launch();
    kern<<<dim3((C + 31) / 32, dm->Hq, dm->B), 256, smem, st>>>(summary, static_cast<const __nv_bfloat16*>(w_up),
                                                                 C, dm->Hq, sb);
  }
  {
    // tcgen05 scorer: q_h and the split chunk rows by TMA (views with 128-byte rows)
    const unsigned long long tokens = (unsigned long long)M, srows = (unsigned long long)dm->B * dm->Hq * C;
    CUtensorMap qmap, smap, spmap, tmap;
    const cuuint64_t qd[4] = {64, tokens, 2, (cuuint64_t)dm->Hq}, qs[3] = {(cuuint64_t)dm->Hq * 256, 128, 256};
    const cuuint32_t qb[4] = {64, ZT_ROWS, 2, 1};
    const cuuint64_t sd[4] = {64, srows, 2, 2}, ss[3] = {768, 256, 128};          // [s_hi | s_lo | ..] rows
    const cuuint32_t sbx[4] = {64, ZT_CH, 2, 2};
    const cuuint64_t pd[3] = {64, srows, 2}, ps[2] = {768, 128};                  // [.. | s'_hi | s'_lo]
    const cuuint32_t pb[3] = {64, ZT_CH, 2};
    const cuuint64_t td[3] = {64, tokens, 2}, ts[2] = {256, 128};                 // [t_hi | t_lo] rows
    const cuuint32_t tb[3] = {64, ZT_ROWS, 2};
    if (!make_tmap_bf16_nd(&qmap, q, 4, qd, qs, qb) || !make_tmap_bf16_nd(&smap, sb, 4, sd, ss, sbx) ||
        !make_tmap_bf16_nd(&spmap, reinterpret_cast<const char*>(sb) + 512, 3, pd, ps, pb) ||
        !make_tmap_bf16_nd(&tmap, tt, 3, td, ts, tb))
      return RDL_ERR_CUDA;
    dim3 grid((C + ZT_CH - 1) / ZT_CH, (dm->Lq + ZT_ROWS - 1) / ZT_ROWS, dm->B * dm->Hkv);
    if (fused_score(dm, RDL_BF16)) {
      // group maxima only, the top-K on them, then the products again for the selected
      // chunks' per-head scores: no per-head score buffer
      if (cudaFuncSetAttribute(zeta_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, ZT_SMEM) !=
              cudaSuccess ||
          cudaFuncSetAttribute(zeta_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, ZT_SMEM) != cudaSuccess)
        return RDL_ERR_CUDA;
      count_launch();
      zeta_tc_kernel<1><<<grid, ZT_THREADS, ZT_SMEM, st>>>(qmap, smap, spmap, tmap, q_pos, entropy, dm->Lq, dm->L,
                                                           dm->Hq, dm->Hkv, dm->w, dm->lambda, nullptr, zeta, nullptr,
                                                           dm->K, nullptr);
      if (cudaGetLastError() != cudaSuccess) return RDL_ERR_CUDA;
      rdl_status s2 = launch_topk(zeta, nullptr, q_pos, dm, idx, z_sel, st);
      if (s2 != RDL_OK) return s2;
      count_launch();
      zeta_tc_kernel<2><<<grid, ZT_THREADS, ZT_SMEM, st>>>(qmap, smap, spmap, tmap, q_pos, entropy, dm->Lq, dm->L,
                                                           dm->Hq, dm->Hkv, dm->w, dm->lambda, nullptr, nullptr, idx,
                                                           dm->K, z_sel);
      return cuda_status(cudaGetLastError());
    }
    if (cudaFuncSetAttribute(zeta_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, ZT_SMEM) != cudaSuccess)
      return RDL_ERR_CUDA;
    count_launch();
    zeta_tc_kernel<0><<<grid, ZT_THREADS, ZT_SMEM, st>>>(qmap, smap, spmap, tmap, q_pos, entropy, dm->Lq, dm->L,
                                                         dm->Hq, dm->Hkv, dm->w, dm->lambda, z_all, zeta, nullptr,
                                                         dm->K, nullptr);
  }
  if (cudaGetLastError() != cudaSuccess) return RDL_ERR_CUDA;
  return launch_topk(zeta, z_all, q_pos, dm, idx, z_sel, st);
}

template <typename T>
rdl_status score_impl(const void* q, const int32_t* q_pos, const void* x, const void* w_down,
                      const void* w_up, const float* summary, const float* entropy,
                      const rdl_dims* dm, int32_t* idx, float* z_sel, void* workspace,
                      cudaStream_t st) {
  const ScoreWs wl = score_ws(dm, std::is_same<T, float>::value ? RDL_F32 : RDL_BF16);
  char* ws = static_cast<char*>(workspace);
  float* t = reinterpret_cast<float*>(ws + wl.t);
  float* qres = reinterpret_cast<float*>(ws + wl.qres);
  float* z_all = reinterpret_cast<float*>(ws + wl.z_all);
  float* zeta = reinterpret_cast<float*>(ws + wl.zeta);
  const int M = dm->B * dm->Lq, N = dm->Hq * dm->d, C = dm->L / S;
  const T* qT = static_cast<const T*>(q);
  if (decode_score_path(dm)) {
    // decode blocks: fused residual query per row, then a tensor-core pass that streams
    // the cached summaries once
    const bool res = dm->r > 0 && x;
    if (cudaFuncSetAttribute(dec_tpart_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_TPART_SMEM) !=
            cudaSuccess ||
        cudaFuncSetAttribute(dec_qres_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_QRES_SMEM) !=
            cudaSuccess ||
        cudaFuncSetAttribute(decode_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DS_SMEM) !=
            cudaSuccess)
      return RDL_ERR_CUDA;
    const int rowblocks = (M + DQ_ROWS - 1) / DQ_ROWS;
    if (res) {
      // t = x W_down by 64-wide slices of D, then summed
      float* tpart = reinterpret_cast<float*>(ws + wl.tpart);
      const int nsl = (dm->D + DQ_KS - 1) / DQ_KS;
      count_launch(2);
      dec_tpart_kernel<T><<<dim3(nsl, rowblocks), 256, DQ_TPART_SMEM, st>>>(
          static_cast<const T*>(x), static_cast<const T*>(w_down), M, dm->D, dm->r, tpart);
      dec_tsum_kernel<<<(M * dm->r + 255) / 256, 256, 0, st>>>(tpart, nsl, M * dm->r, t);
    }
    count_launch(2);
    dec_qres_kernel<T><<<dim3((N + 127) / 128, rowblocks), 256, DQ_QRES_SMEM, st>>>(
        qT, res ? t : nullptr, static_cast<const T*>(w_up), M, res ? dm->r : 0, N, qres);
    decode_score_kernel<<<dim3((C + DS_CH - 1) / DS_CH, dm->B * dm->Hkv), 128, DS_SMEM, st>>>(
        qres, q_pos, summary, entropy, dm->Lq, dm->L, dm->Hq, dm->Hkv, dm->w, dm->lambda, z_all, zeta);
    if (cudaGetLastError() != cudaSuccess) return RDL_ERR_CUDA;
    return launch_topk(zeta, z_all, q_pos, dm, idx, z_sel, st);
  }
  if (dm->r > 0 && x) {
    count_launch(2);
    if (M <= 64) {
      smallm_gemm_kernel<T, T><<<dim3((dm->r + 31) / 32, M), 256, 0, st>>>(
          static_cast<const T*>(x), static_cast<const T*>(w_down), t, M, dm->r, dm->D);
    } else {
      dim3 g1((dm->r + 63) / 64, (M + 63) / 64);
      gemm_f32_kernel<T, T, T><<<g1, 256, 0, st>>>(static_cast<const T*>(x), static_cast<const T*>(w_down),
                                                   (const T*)nullptr, t, M, dm->r, dm->D);
    }
    dim3 g2((N + 63) / 64, (M + 63) / 64);
    gemm_f32_kernel<float, T, T><<<g2, 256, 0, st>>>(t, static_cast<const T*>(w_up), qT, qres, M, N, dm->r);
  } else {
    // no residual: q_res = q (an r = 0 product adds nothing)
    count_launch();
    dim3 g2((N + 63) / 64, (M + 63) / 64);
    gemm_f32_kernel<float, T, T><<<g2, 256, 0, st>>>(t, static_cast<const T*>(w_up), qT, qres, M, N, 0);
  }
  dim3 g3((C + 63) / 64, (dm->Lq + 63) / 64, dm->B * dm->Hkv);
  count_launch();    // zeta (top-K counted in launch_topk)
  if (dm->d == 128)
    zeta_kernel<128><<<g3, 256, 0, st>>>(qres, q_pos, summary, entropy, dm->Lq, dm->L, dm->Hq, dm->Hkv,
                                         dm->w, dm->lambda, z_all, zeta);
  else
    zeta_kernel<64><<<g3, 256, 0, st>>>(qres, q_pos, summary, entropy, dm->Lq, dm->L, dm->Hq, dm->Hkv,
                                        dm->w, dm->lambda, z_all, zeta);
  if (cudaGetLastError() != cudaSuccess) return RDL_ERR_CUDA;
  return launch_topk(zeta, z_all, q_pos, dm, idx, z_sel, st);
}

template <typename T, bool ROUTE>
rdl_status generic_attn(const void* q, const int32_t* q_pos, const void* k, const void* v,
                        const int32_t* idx, const float* z_sel, const rdl_dims* dm, void* o,
                        float* lse, cudaStream_t st) {
  dim3 grid(dm->Lq, dm->Hkv, dm->B);
  count_launch();
  const T *qT = static_cast<const T*>(q), *kT = static_cast<const T*>(k), *vT = static_cast<const T*>(v);
  if (dm->d == 128)
    generic_attn_kernel<T, 128, ROUTE><<<grid, 128, 0, st>>>(qT, q_pos, kT, vT, idx, z_sel, dm->L, dm->Lq,
                                                            dm->Hq, dm->Hkv, dm->K, dm->w, dm->flags,
                                                            static_cast<T*>(o), lse);
  else
    generic_attn_kernel<T, 64, ROUTE><<<grid, 128, 0, st>>>(qT, q_pos, kT, vT, idx, z_sel, dm->L, dm->Lq,
                                                           dm->Hq, dm->Hkv, dm->K, dm->w, dm->flags,
                                                           static_cast<T*>(o), lse);
  return cuda_status(cudaGetLastError());
}

template <int MODE>
rdl_status launch_window_mma(const void* q, const int32_t* q_pos, const void* k, const void* v,
                             const rdl_dims* dm, void* o, float* lse, float* o_loc, float* lam_loc,
                             int nsplit, cudaStream_t st) {
  const int G = dm->Hq / dm->Hkv;
  if (nsplit == 1 && dm->w >= 0 && G <= 8) {
    // one key range per tile: the tcgen05 kernel (16 tokens x 8 head slots per CTA)
    CUtensorMap qmap, kmap, vmap;
    const unsigned long long tokens = (unsigned long long)dm->B * dm->Lq;
    const unsigned long long kvrows = (unsigned long long)dm->B * dm->Hkv * dm->L;
    if (!make_tmap_q_run(&qmap, q, tokens, (unsigned)dm->Hq, WT_TOK) ||
        !make_tmap_kv_halves(&kmap, k, kvrows, WT_KEYS) || !make_tmap_kv_halves(&vmap, v, kvrows, WT_KEYS))
      return RDL_ERR_CUDA;
    auto tk = window_tc_kernel<MODE>;
    if (cudaFuncSetAttribute(tk, cudaFuncAttributeMaxDynamicSharedMemorySize, WT_SMEM) != cudaSuccess)
      return RDL_ERR_CUDA;
    dim3 grid((dm->Lq + WT_TOK - 1) / WT_TOK, dm->B * dm->Hkv);
    count_launch();
    tk<<<grid, WT_THREADS, WT_SMEM, st>>>(qmap, kmap, vmap, q_pos, dm->L, dm->Lq, dm->Hq, dm->Hkv, dm->w,
                                          static_cast<__nv_bfloat16*>(o), lse, o_loc, lam_loc);
    return cuda_status(cudaGetLastError());
  }
  const size_t smem = window_mma_smem(G);
  auto kern = window_mma_kernel<MODE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return RDL_ERR_CUDA;
  dim3 grid((dm->Lq + WIN_ROWS - 1) / WIN_ROWS, dm->B * dm->Hkv, nsplit);
  count_launch();
  kern<<<grid, 32 * G, smem, st>>>(static_cast<const __nv_bfloat16*>(q), q_pos,
                                   static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                                   dm->L, dm->Lq, dm->Hq, dm->Hkv, dm->w, static_cast<__nv_bfloat16*>(o), lse,
                                   o_loc, lam_loc, nsplit);
  return cuda_status(cudaGetLastError());
}

rdl_status attn_chunk_major(const void* q, const int32_t* q_pos, const void* k, const void* v, const int32_t* idx,
                            const float* z_sel, const rdl_dims* dm, void* o, float* lse, void* workspace,
                            cudaStream_t st) {
  const AttnWs wl = attn_ws(dm, RDL_BF16);
  char* ws = static_cast<char*>(workspace);
  float* o_loc = reinterpret_cast<float*>(ws + wl.o_loc);
  float* lam_loc = reinterpret_cast<float*>(ws + wl.lam_loc);
  int* counts = reinterpret_cast<int*>(ws + wl.counts);
  int* cursor = reinterpret_cast<int*>(ws + wl.cursor);
  int* nitems = reinterpret_cast<int*>(ws + wl.nitems);
  int* offs = reinterpret_cast<int*>(ws + wl.offs);
  int* list = reinterpret_cast<int*>(ws + wl.list);
  CmItem* items = reinterpret_cast<CmItem*>(ws + wl.items);
  __half* part = reinterpret_cast<__half*>(ws + wl.part);
  const int C = dm->L / S, BG = dm->B * dm->Hkv;
  // the local window: normalised output and log-sum-exp per (row, head)
  const int nsw = window_splits(dm);
  rdl_status s = launch_window_mma<1>(q, q_pos, k, v, dm, nullptr, nullptr, o_loc, lam_loc, nsw, st);
  if (s != RDL_OK) return s;
  // buckets of selections per (batch, group, chunk) and the work items
  if (cudaMemsetAsync(ws + wl.zero, 0, wl.zero_bytes, st) != cudaSuccess) return RDL_ERR_CUDA;
  const dim3 bgrid((dm->Lq + CM_ROWS - 1) / CM_ROWS, BG);
  if (cudaFuncSetAttribute(cm_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C * 4) != cudaSuccess ||
      cudaFuncSetAttribute(cm_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * C * 4) != cudaSuccess ||
      cudaFuncSetAttribute(cm_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, CM_SMEM) != cudaSuccess)
    return RDL_ERR_CUDA;
  count_launch(5);
  cm_count_kernel<<<bgrid, 512, C * 4, st>>>(idx, q_pos, dm->Lq, dm->L, dm->Hkv, dm->K, dm->w, dm->flags, counts);
  cm_scan_kernel<<<BG, 1024, 0, st>>>(counts, C, offs, nitems, items);
  cm_scatter_kernel<<<bgrid, 512, 2 * C * 4, st>>>(idx, q_pos, dm->Lq, dm->L, dm->Hkv, dm->K, dm->w, dm->flags, offs,
                                                  cursor, list);
  // chunk passes: persistent CTAs, one per SM
  CUtensorMap kmap, vmap, qmap;
  const unsigned long long kvrows = (unsigned long long)dm->B * dm->Hkv * dm->L;
  if (!make_tmap_kv_halves(&kmap, k, kvrows) || !make_tmap_kv_halves(&vmap, v, kvrows) ||
      !make_tmap_q_run(&qmap, q, (unsigned long long)dm->B * dm->Lq, (unsigned)dm->Hq, 1))
    return RDL_ERR_CUDA;
  const size_t mi = cm_max_items(dm);
  const int grid = (int)(mi < (size_t)kSMs ? mi : (size_t)kSMs);
  cm_attn_kernel<<<grid, CM_THREADS, CM_SMEM, st>>>(kmap, vmap, qmap, items, nitems,
                                                   list, dm->Lq, dm->L, dm->Hq, dm->Hkv, dm->K, dm->flags, part);
  const long long n = (long long)dm->B * dm->Lq * dm->Hq;
  cm_combine_kernel<<<(unsigned)((n + CM_COMB_WARPS - 1) / CM_COMB_WARPS), CM_COMB_WARPS * 32, 0, st>>>(q_pos, idx, z_sel, part, o_loc, lam_loc, nsw, dm->B, dm->L,
                                                             dm->Lq, dm->Hq, dm->Hkv, dm->K, dm->w, dm->flags,
                                                             static_cast<__nv_bfloat16*>(o), lse);
  return cuda_status(cudaGetLastError());
}

}  // namespace

extern "C" {

const char* rdl_version(void) { return "0.1.0"; }

unsigned long long rdl_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* rdl_status_string(rdl_status s) {
  switch (s) {
    case RDL_OK: return "ok";
    case RDL_ERR_INVALID_ARG: return "invalid argument";
    case RDL_ERR_UNSUPPORTED: return "unsupported combination";
    case RDL_ERR_CUDA: return "CUDA error";
    case RDL_ERR_TIMEOUT: return "device wait timed out";
    case RDL_ERR_WORKSPACE: return "workspace too small";
    case RDL_ERR_DEVICE_CHECK: return "device-side check failed";
    case RDL_ERR_SCRATCH_LIMIT: return "size exceeds the static scratch of the no-allocation entry point";
  }
  return "unknown status";
}

size_t rdl_workspace_bytes(int which, const rdl_dims* dims, rdl_dtype dtype) {
  if (!route_dims_ok(dims) || !dtype_ok(dtype)) return 0;
  const rdl_dims dm = clamp_w(dims);     // the calls size their workspace on the clamped radius
  if (which == RDL_WS_SCORE) return score_ws(&dm, dtype).total;
  if (which == RDL_WS_ATTN) return attn_ws(&dm, dtype).total;
  if (which == RDL_WS_SWA) return swa_ws(&dm, dtype);
  return 0;
}

rdl_status rdl_summary_pool(const void* q_mask, long long q_chunk_stride, long long q_batch_stride,
                            const void* k, const void* v, const rdl_dims* dims, rdl_dtype dtype,
                            float* summary, float* entropy, void* o_mask, void* stream) {
  if (!dims_ok(dims) || !dtype_ok(dtype)) return RDL_ERR_INVALID_ARG;
  if (!q_mask || !k || !summary || !entropy) return RDL_ERR_INVALID_ARG;
  if (o_mask && !v) return RDL_ERR_INVALID_ARG;
  if (!aligned16(q_mask) || !aligned16(k) || (v && !aligned16(v)) || !aligned16(summary) ||
      (o_mask && !aligned16(o_mask)))
    return RDL_ERR_INVALID_ARG;
  const long long row = (long long)dims->Hq * dims->d;
  if (q_chunk_stride < row || q_batch_stride < 0) return RDL_ERR_INVALID_ARG;
  const cudaStream_t st = as_stream(stream);
  cudaError_t e;
  if (dtype == RDL_BF16) {
    e = dims->d == 128 ? launch_summary_pool<__nv_bfloat16, 128>(q_mask, q_chunk_stride, q_batch_stride, k, v,
                                                                 *dims, summary, entropy, o_mask, st)
                       : launch_summary_pool<__nv_bfloat16, 64>(q_mask, q_chunk_stride, q_batch_stride, k, v,
                                                                *dims, summary, entropy, o_mask, st);
  } else {
    e = dims->d == 128 ? launch_summary_pool<float, 128>(q_mask, q_chunk_stride, q_batch_stride, k, v, *dims,
                                                         summary, entropy, o_mask, st)
                       : launch_summary_pool<float, 64>(q_mask, q_chunk_stride, q_batch_stride, k, v, *dims,
                                                        summary, entropy, o_mask, st);
  }
  return cuda_status(e);
}

rdl_status rdl_route_score_topk(const void* q, const int32_t* q_pos, const void* x,
                                const void* w_down, const void* w_up, const float* summary,
                                const float* entropy, const rdl_dims* dims, rdl_dtype dtype,
                                int32_t* idx, float* z_sel, void* workspace, size_t ws_bytes,
                                void* stream) {
  if (!route_dims_ok(dims) || !dtype_ok(dtype)) return RDL_ERR_INVALID_ARG;
  if (!q_pos && dims->Lq != dims->L) return RDL_ERR_INVALID_ARG;
  if (dims->L / S > kMaxC) return RDL_ERR_UNSUPPORTED;
  const bool residual = dims->r > 0 && x != nullptr;
  if (!q || !summary || !entropy || !idx || !z_sel || !workspace) return RDL_ERR_INVALID_ARG;
  if (residual && (!w_down || !w_up)) return RDL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(summary) || !aligned16(entropy) || !aligned16(idx) ||
      !aligned16(z_sel) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (residual && (!aligned16(x) || !aligned16(w_down) || !aligned16(w_up))) ||
      (q_pos && !aligned16(q_pos)))
    return RDL_ERR_INVALID_ARG;
  rdl_dims dm = clamp_w(dims);
  if (!residual) dm.r = 0;
  if (ws_bytes < score_ws(&dm, dtype).total) return RDL_ERR_WORKSPACE;
  const cudaStream_t st = as_stream(stream);
  if (dec_score_ok(&dm, dtype))
    return score_decode(q, q_pos, x, w_down, w_up, summary, entropy, &dm, idx, z_sel, workspace, st);
  if (dm.flags & RDL_FLAG_SPLIT_SUMMARY) return RDL_ERR_UNSUPPORTED;
  if (fast_score(&dm, dtype))
    return score_fast(q, q_pos, x, w_down, w_up, summary, entropy, &dm, idx, z_sel, workspace, st);
  return dtype == RDL_BF16 ? score_impl<__nv_bfloat16>(q, q_pos, x, w_down, w_up, summary, entropy, &dm, idx,
                                                       z_sel, workspace, st)
                           : score_impl<float>(q, q_pos, x, w_down, w_up, summary, entropy, &dm, idx, z_sel,
                                               workspace, st);
}

rdl_status rdl_route_attn(const void* q, const int32_t* q_pos, const void* k, const void* v,
                          const int32_t* idx, const float* z_sel, const rdl_dims* dims,
                          rdl_dtype dtype, void* o, float* lse, void* workspace, size_t ws_bytes,
                          void* stream) {
  if (!route_dims_ok(dims) || !dtype_ok(dtype)) return RDL_ERR_INVALID_ARG;
  if (!q_pos && dims->Lq != dims->L) return RDL_ERR_INVALID_ARG;
  if (!q || !k || !v || !idx || !z_sel || !o) return RDL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(z_sel) ||
      !aligned16(o) || (lse && !aligned16(lse)) || (q_pos && !aligned16(q_pos)))
    return RDL_ERR_INVALID_ARG;
  const cudaStream_t st = as_stream(stream);
  const rdl_dims dmc = clamp_w(dims);
  dims = &dmc;
  if (!fast_attn(dims, dtype)) {
    return dtype == RDL_BF16 ? generic_attn<__nv_bfloat16, true>(q, q_pos, k, v, idx, z_sel, dims, o, lse, st)
                             : generic_attn<float, true>(q, q_pos, k, v, idx, z_sel, dims, o, lse, st);
  }
  const AttnWs wl = attn_ws(dims, dtype);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return RDL_ERR_INVALID_ARG;
  if (ws_bytes < wl.total) return RDL_ERR_WORKSPACE;
  if (dec_attn_ok(dims, dtype) && dec_attn_stages(dims, dims->K) > 0)
    return attn_decode(q, q_pos, k, v, idx, z_sel, dims, o, lse, workspace, st);
  if (use_chunk_major(dims, dtype)) return attn_chunk_major(q, q_pos, k, v, idx, z_sel, dims, o, lse, workspace, st);
  char* ws = static_cast<char*>(workspace);
  float* o_loc = reinterpret_cast<float*>(ws + wl.o_loc);
  float* lam_loc = reinterpret_cast<float*>(ws + wl.lam_loc);
  float* o_acc = reinterpret_cast<float*>(ws + wl.o_acc);
  const int nsw = window_splits(dims);
  rdl_status s = launch_window_mma<1>(q, q_pos, k, v, dims, nullptr, nullptr, o_loc, lam_loc, nsw, st);
  if (s != RDL_OK) return s;
  const int ns = attn_splits(dims);
  const size_t rows = (size_t)dims->B * dims->Lq * dims->Hq;
  const int C = dims->L / S;
  if (ns == 1 && C <= CT_MAXC && dims->K <= CT_MAXK) {
    // prefill: tcgen05 kernel, 48-row tiles sharing each selected chunk's K/V
    CtMaps maps;                                    // copied into the launch parameters
    const unsigned long long tokens = (unsigned long long)dims->B * dims->Lq;
    const unsigned long long kvrows = (unsigned long long)dims->B * dims->Hkv * dims->L;
    bool mapped = make_tmap_kv_halves(&maps.k, k, kvrows) && make_tmap_kv_halves(&maps.v, v, kvrows);
    for (unsigned r = 1; r <= 8 && mapped; ++r) mapped = make_tmap_q_run(&maps.q[r - 1], q, tokens, dims->Hq, r);
    if (mapped) {
      if (cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, CT_SMEM) !=
          cudaSuccess)
        return RDL_ERR_CUDA;
      dim3 grid((dims->Lq + CT_TQ - 1) / CT_TQ, dims->B * dims->Hkv);
      count_launch();
      chunk_tc_kernel<<<grid, CT_THREADS, CT_SMEM, st>>>(maps, q_pos, idx, z_sel, o_loc, lam_loc, nsw, dims->L,
                                                         dims->Lq, dims->Hq, dims->Hkv, dims->K, dims->w,
                                                         dims->flags, static_cast<__nv_bfloat16*>(o), lse);
      return cuda_status(cudaGetLastError());
    }
  }
  const size_t smem = (size_t)CH_WARPS * CH_WARP_SMEM;
  if (cudaFuncSetAttribute(chunk_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return RDL_ERR_CUDA;
  const long long warps = (long long)dims->Lq * dims->Hkv * ns;
  dim3 grid((unsigned)((warps + CH_WARPS - 1) / CH_WARPS), dims->B);
  count_launch(ns > 1 ? 2 : 1);
  chunk_mma_kernel<<<grid, CH_WARPS * 32, smem, st>>>(
      static_cast<const __nv_bfloat16*>(q), q_pos, static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), idx, z_sel, o_loc, lam_loc, dims->L, dims->Lq, dims->Hq, dims->Hkv,
      dims->K, dims->w, ns, dims->flags, static_cast<__nv_bfloat16*>(o), lse, o_acc, nsw);
  if (cudaGetLastError() != cudaSuccess) return RDL_ERR_CUDA;
  if (ns > 1) {
    const long long n = (long long)rows * dims->d;
    const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    chunk_finalize_kernel<<<blocks, 256, 0, st>>>(o_acc, ns, q_pos, dims->Lq, dims->Hq * dims->d, dims->B,
                                                  static_cast<__nv_bfloat16*>(o));
    if (cudaGetLastError() != cudaSuccess) return RDL_ERR_CUDA;
  }
  return RDL_OK;
}

rdl_status rdl_swa_attn(const void* q, const int32_t* q_pos, const void* k, const void* v,
                        const rdl_dims* dims, rdl_dtype dtype, void* o, float* lse, void* workspace,
                        size_t ws_bytes, void* stream) {
  if (!dims_ok(dims) || !dtype_ok(dtype) || dims->w < 0) return RDL_ERR_INVALID_ARG;
  if (!q_pos && dims->Lq != dims->L) return RDL_ERR_INVALID_ARG;
  if (!q || !k || !v || !o) return RDL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)) ||
      (q_pos && !aligned16(q_pos)))
    return RDL_ERR_INVALID_ARG;
  const cudaStream_t st = as_stream(stream);
  const rdl_dims dmc = clamp_w(dims);
  dims = &dmc;
  if (!fast_attn(dims, dtype)) {
    return dtype == RDL_BF16 ? generic_attn<__nv_bfloat16, false>(q, q_pos, k, v, nullptr, nullptr, dims, o, lse, st)
                             : generic_attn<float, false>(q, q_pos, k, v, nullptr, nullptr, dims, o, lse, st);
  }
  const size_t need = swa_ws(dims, dtype);
  if (dec_swa_ok(dims, dtype)) {
    // decode blocks: one launch, one CTA per (b, group, pair of rows); no workspace
    const unsigned long long kvrows = (unsigned long long)dims->B * dims->Hkv * dims->L;
    CUtensorMap kmap, vmap;
    if (!make_tmap_kv_halves(&kmap, k, kvrows) || !make_tmap_kv_halves(&vmap, v, kvrows)) return RDL_ERR_CUDA;
    const int smem = dec::swa_smem();
    if (cudaFuncSetAttribute(dec::dec_swa_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return RDL_ERR_CUDA;
    const float sl2 = (float)(1.0 / sqrt((double)dims->d) * 1.4426950408889634);
    const int ctas = dims->B * dims->Hkv * ((dims->Lq + 1) / 2);
    if (launch_pdl(dec::dec_swa_kernel<false>, dim3(ctas), dim3(dec::SW_WARPS * 32), smem, st, kmap, vmap,
                   static_cast<const __nv_bfloat16*>(q), q_pos, dims->L, dims->Lq, dims->Hq, dims->Hkv, dims->w, sl2,
                   static_cast<__nv_bfloat16*>(o), lse, (float*)nullptr, (float2*)nullptr) != cudaSuccess)
      return RDL_ERR_CUDA;
    return RDL_OK;
  }
  if (need == 0 || !workspace) return launch_window_mma<0>(q, q_pos, k, v, dims, o, lse, nullptr, nullptr, 1, st);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return RDL_ERR_INVALID_ARG;
  if (ws_bytes < need) return RDL_ERR_WORKSPACE;
  // few rows: key-split partials, then the combine pass
  const int nsw = window_splits(dims);
  const size_t rows = (size_t)dims->B * dims->Lq * dims->Hq;
  float* o_part = static_cast<float*>(workspace);
  float* l_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(sizeof(float) * rows * dims->d * nsw));
  rdl_status s = launch_window_mma<0>(q, q_pos, k, v, dims, nullptr, nullptr, o_part, l_part, nsw, st);
  if (s != RDL_OK) return s;
  const long long n = (long long)rows * dims->d;
  const int blocks = (int)((n + 255) / 256 < 2048 ? (n + 255) / 256 : 2048);
  count_launch();
  window_combine_kernel<<<blocks, 256, 0, st>>>(o_part, l_part, nsw, dims->B, dims->Lq, dims->Hq,
                                                static_cast<__nv_bfloat16*>(o), lse);
  return cuda_status(cudaGetLastError());
}

rdl_status rdl_last_device_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return RDL_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return RDL_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return RDL_ERR_CUDA;
  return static_cast<rdl_status>(v);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// rdl_route_attn_noalloc: rdl_route_attn with a library-held static scratch array, for
// hosts that cannot hand the library device memory at call time (engines that plan all
// device buffers before serving, plugin interfaces without an allocator).  It forwards to
// rdl_route_attn with the array as the workspace; no allocation anywhere on this path.
namespace {

constexpr size_t kNoAllocScratchBytes = RDL_NOALLOC_SCRATCH_BYTES;
// One copy per device that loads the library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
// (context id, address) per device: the address belongs to the module loaded into one
// context, and context ids are unique for the life of the process, so a new primary context
// on the device (after cudaDeviceReset) triggers a fresh lookup.
struct NoAllocSlot {
  unsigned long long ctx_id = 0;
  void* ptr = nullptr;
};
NoAllocSlot g_noalloc_slot[kMaxDevices];
std::mutex g_noalloc_mu;

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}
// Id of the current context, 0 when none is current.
unsigned long long current_context_id() {
  typedef int (*CtxGetCurrentFn)(void**);                        // cuCtxGetCurrent
  typedef int (*CtxGetIdFn)(void*, unsigned long long*);         // cuCtxGetId
  static const CtxGetCurrentFn get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  void* ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != 0 || !ctx || get_id(ctx, &id) != 0) return 0;
  return id;
}

// Device address of the scratch array on the current device.  In host code the array's
// name is only a host-side stand-in, so the address must come from cudaGetSymbolAddress,
// looked up with that device current: on the first call on that device, and again whenever
// the device's context has changed since the last lookup.
void* noalloc_scratch_ptr() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocSlot& slot = g_noalloc_slot[dev];
  unsigned long long id = current_context_id();     // 0 until the runtime has touched this device
  if (id && slot.ptr && slot.ctx_id == id) return slot.ptr;
  void* p = nullptr;
  // also creates and binds the device's primary context when none is current yet
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
  id = current_context_id();
  if (!id) return nullptr;
  slot.ctx_id = id;
  slot.ptr = p;
  return p;
}

}  // namespace

extern "C" rdl_status rdl_route_attn_noalloc(const void* q, const int32_t* q_pos, const void* k,
                                             const void* v, const int32_t* idx, const float* z_sel,
                                             const rdl_dims* dims, rdl_dtype dtype, void* o,
                                             float* lse, void* stream) {
  if (!route_dims_ok(dims) || !dtype_ok(dtype)) return RDL_ERR_INVALID_ARG;
  const rdl_dims dmc = clamp_w(dims);
  if (attn_ws(&dmc, dtype).total > kNoAllocScratchBytes) return RDL_ERR_SCRATCH_LIMIT;
  void* scratch = noalloc_scratch_ptr();
  if (!scratch) return RDL_ERR_CUDA;
  return rdl_route_attn(q, q_pos, k, v, idx, z_sel, dims, dtype, o, lse, scratch,
                        kNoAllocScratchBytes, stream);
}
