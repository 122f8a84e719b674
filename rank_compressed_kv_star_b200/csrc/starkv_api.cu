// C-ABI entry points of libstarkv: argument validation, launch planning,
// workspace layout and launch sequencing on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <tuple>
#include <mutex>
#include <utility>

#include "../../include/starkv.h"
#include "append_kernels.cuh"
#include "decode_kernels.cuh"

// Launch-shape defaults (overridable at build time for tuning sweeps).
#ifndef STARKV_K_CTAS_PER_SM
#define STARKV_K_CTAS_PER_SM 1
#endif
#ifndef STARKV_K_STAGE_CAP
#define STARKV_K_STAGE_CAP 65536
#endif
#ifndef STARKV_KTC_CTAS_PER_SM
#define STARKV_KTC_CTAS_PER_SM 3
#endif
#ifndef STARKV_KTC_SMEM_BYTES
#define STARKV_KTC_SMEM_BYTES (224 * 1024)   // shared memory of the K-pass CTAs on one SM (228 KB less 1 KB per CTA)
#endif
#ifndef STARKV_K_RING_BYTES
#define STARKV_K_RING_BYTES (200 * 1024 / STARKV_K_CTAS_PER_SM)
#endif
#ifndef STARKV_V_RRANGE
#define STARKV_V_RRANGE 1024
#endif
#ifndef STARKV_CV_STAGE_CAP
#define STARKV_CV_STAGE_CAP 8   // ring stages of the chunked-prefill V pass
#endif
#ifndef STARKV_CV_LW_MAX
#define STARKV_CV_LW_MAX 256    // widest group of virtual heads of one chunked-prefill V-pass CTA
#endif
#ifndef STARKV_CV_PPS
#define STARKV_CV_PPS 4         // pages per ring stage of the chunked-prefill V pass (at most)
#endif
#ifndef STARKV_V_PPS
#define STARKV_V_PPS 1          // pages per ring stage of the decode V pass (at most)
#endif
#ifndef STARKV_K_CHUNK_BYTES
#define STARKV_K_CHUNK_BYTES (1024 * 1024)   // codes per chunk of pages handed out by the K pass's counter
#endif
#ifndef STARKV_V_MIN_PAGES
#define STARKV_V_MIN_PAGES 16   // fewest pages per decode V-pass CTA when a call has few pages
#endif
#ifndef STARKV_APP_KS_MAX
#define STARKV_APP_KS_MAX 4     // largest cluster splitting the V-code GEMM's K range
#endif
#ifndef STARKV_V_RING_BYTES
#define STARKV_V_RING_BYTES (105 * 1024)
#endif

namespace starkv {
namespace {

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return 148; }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int kv_heads(const starkv_layer_desc* d) { return d->num_kv_heads > 0 ? d->num_kv_heads : d->num_heads; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int pow2_ceil(int x) { int p = 1; while (p < x) p <<= 1; return p; }

starkv_status check_desc(const starkv_layer_desc* d) {
  if (!d) return STARKV_ERR_INVALID_ARG;
  if (d->num_heads <= 0 || d->head_dim <= 0 || d->k_rank <= 0 || d->v_rank <= 0 || d->num_blocks <= 0 ||
      d->max_blocks_per_seq <= 0)
    return STARKV_ERR_INVALID_ARG;
  if (d->block_size != 16) return STARKV_ERR_UNSUPPORTED;
  if (!is_pow2(d->num_heads) || d->num_heads > 64) return STARKV_ERR_UNSUPPORTED;
  if (d->num_kv_heads < 0) return STARKV_ERR_INVALID_ARG;
  if (d->num_kv_heads > 0 && (!is_pow2(d->num_kv_heads) || d->num_kv_heads > d->num_heads))
    return STARKV_ERR_UNSUPPORTED;
  if (!(d->head_dim == 32 || d->head_dim == 64 || d->head_dim == 128 || d->head_dim == 256))
    return STARKV_ERR_UNSUPPORTED;
  if (d->k_rank % 16 != 0 || d->k_rank > 256) return STARKV_ERR_UNSUPPORTED;
  if (d->v_rank % 64 != 0 || d->v_rank > 8192) return STARKV_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->num_blocks) * 16 > INT32_MAX) return STARKV_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->max_blocks_per_seq) * 16 > INT32_MAX) return STARKV_ERR_UNSUPPORTED;
  return STARKV_OK;
}

// ------------------------------------------------------------------ planning
struct DecodePlan {
  int H, Hkv, log2G, d, r, R, B, MB, NB, cap, n_pages_max, t_pad, npad;
  // K pass
  int L, CPT, log2H, tps, k_stages, k_ctas, k_chunk_pages;
  uint32_t k_stage_bytes;
  size_t k_smem;
  // K pass on tensor cores (grouped queries)
  bool ktc;
  int ktc_log2tpt, ktc_ksteps, ktc_kb, ktc_nmma, ktc_brows, ktc_nacc, ktc_nbs, ktc_stages;
  uint32_t ktc_a_bytes, ktc_b_bytes, ktc_tmem;
  size_t ktc_smem;
  // V pass
  int n_rr, r_range, r_range_pad, n_chunks, n_mtiles, v_stages, v_ctas, v_per_sm, v_pps;
  uint32_t vtile, ltile, ptile, tmem_cols;
  size_t v_smem;
  // finish: Z / L from the partials and the up-projection (tcgen05, split-K cluster)
  int up_mt, up_bt_rows, up_bt, up_npad, up_ks, up_kpc, up_stages, up_zrows;
  uint32_t up_stage_bytes, up_tmem;
  size_t up_smem;
  starkv_workspace_layout ws;
};

// Threads per (token, head) dot product and 16-byte chunks per thread.
void plan_kpass_shape(int r, int* L, int* CPT) {
  const int cp = r / 8;
  if (cp <= 4) { *L = 1; *CPT = 4; }        // r <= 32
  else if (cp <= 8) { *L = 1; *CPT = 8; }   // r <= 64
  else if (cp <= 12) { *L = 1; *CPT = 12; } // r <= 96
  else if (cp <= 16) { *L = 2; *CPT = 8; }  // r <= 128
  else { *L = 4; *CPT = 8; }                // r <= 256
}

// ------------------------------------------------------ kernel attributes
// Raises a kernel's dynamic shared-memory limit once per (kernel, device), and
// again only when a larger size is needed.
template <typename K>
bool set_smem(K kernel, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> set_bytes;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return false; }
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  std::lock_guard<std::mutex> lock(mu);
  auto it = set_bytes.find(key);
  if (it != set_bytes.end() && it->second >= static_cast<int>(bytes)) return true;
  // the largest shared-memory carveout, so that as many CTAs as the plan
  // counts on fit on one SM
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
          cudaSuccess ||
      cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           static_cast<int>(cudaSharedmemCarveoutMaxShared)) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  set_bytes[key] = static_cast<int>(bytes);
  return true;
}

// Registers per thread of the tensor-core K pass instance <G, H> (0 if unknown).
template <int G, int H>
int ktc_regs() {
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kpass_tc_kernel<G, H>) != cudaSuccess) { cudaGetLastError(); return 0; }
  return fa.numRegs;
}

template <int H>
int ktc_regs_h(int log2G) {
  switch (log2G) {
    case 1: if constexpr (H / 2 <= 16) return ktc_regs<2, H>(); break;
    case 2: if constexpr (H >= 4 && H / 4 <= 16) return ktc_regs<(H >= 4 ? 4 : H), H>(); break;
    case 3: if constexpr (H >= 8) return ktc_regs<(H >= 8 ? 8 : H), H>(); break;
    case 4: if constexpr (H >= 16) return ktc_regs<(H >= 16 ? 16 : H), H>(); break;
    case 5: if constexpr (H >= 32) return ktc_regs<(H >= 32 ? 32 : H), H>(); break;
    case 6: if constexpr (H >= 64) return ktc_regs<(H >= 64 ? 64 : H), H>(); break;
    default: break;
  }
  return 0;
}

int ktc_num_regs(int log2G, int H) {
  switch (H) {
    case 8: return ktc_regs_h<8>(log2G);
    case 16: return ktc_regs_h<16>(log2G);
    case 32: return ktc_regs_h<32>(log2G);
    case 64: return ktc_regs_h<64>(log2G);
    default: return 0;
  }
}

starkv_status make_plan(const starkv_layer_desc* d, int32_t batch, int32_t max_seq_len, DecodePlan* pl) {
  starkv_status st = check_desc(d);
  if (st != STARKV_OK) return st;
  if (batch < 0 || max_seq_len < 0) return STARKV_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_seq_len) > static_cast<int64_t>(d->max_blocks_per_seq) * 16)
    return STARKV_ERR_INVALID_ARG;
  DecodePlan& p = *pl;
  std::memset(&p, 0, sizeof(p));
  p.H = d->num_heads; p.d = d->head_dim; p.r = d->k_rank; p.R = d->v_rank;
  p.Hkv = kv_heads(d);
  p.log2G = 0;
  while ((p.Hkv << p.log2G) < p.H) ++p.log2G;
  p.B = batch; p.MB = d->max_blocks_per_seq; p.NB = d->num_blocks;
  p.cap = max_seq_len;
  p.n_pages_max = (max_seq_len + 15) / 16;
  p.t_pad = p.n_pages_max * 16;
  p.npad = p.H < 16 ? 16 : p.H;
  const int sms = device_sm_count();

  // K pass: ring stages of whole tokens, up to one whole 16-token page per bulk
  // copy (64 KiB at H=32, r=64: large copies measured fastest), ~200 KiB of
  // ring, one CTA per SM
  plan_kpass_shape(p.r, &p.L, &p.CPT);
  p.log2H = 0;
  while ((1 << p.log2H) < p.H) ++p.log2H;
  const uint32_t tok = static_cast<uint32_t>(p.Hkv) * p.r * 2;   // code bytes per token
  p.tps = 16;
  while (p.tps > 1 && p.tps * tok > static_cast<uint32_t>(STARKV_K_STAGE_CAP)) p.tps >>= 1;
  // small pages: several whole pages per stage (up to 8), same byte budget
  while (p.tps >= 16 && p.tps < 128 && 2u * p.tps * tok <= static_cast<uint32_t>(STARKV_K_STAGE_CAP)) p.tps <<= 1;
  p.k_stage_bytes = p.tps * tok;
  p.k_stages = static_cast<int>(static_cast<uint32_t>(STARKV_K_RING_BYTES) / p.k_stage_bytes);
  if (p.k_stages > 8) p.k_stages = 8;
  if (p.k_stages < 2) p.k_stages = 2;
  p.k_smem = static_cast<size_t>(p.k_stages) * p.k_stage_bytes + p.k_stages * sizeof(StageMeta) +
             2 * p.k_stages * sizeof(uint64_t);
  p.k_ctas = sms * STARKV_K_CTAS_PER_SM;
  // pages per chunk handed out by the K pass's counter: about 1 MiB of codes (smaller chunks
  // balance better but make a CTA change sequence, and reload its queries, more often),
  // and at least four chunks per CTA when the call has few pages
  p.k_chunk_pages = static_cast<int>(static_cast<uint32_t>(STARKV_K_CHUNK_BYTES) / (16u * tok));
  {
    const int64_t pages_max = static_cast<int64_t>(batch) * ((p.cap + 15) / 16);
    const int64_t per_cta =
        (pages_max + 4 * static_cast<int64_t>(p.k_ctas) - 1) / (4 * static_cast<int64_t>(p.k_ctas));
    if (per_cta < p.k_chunk_pages) p.k_chunk_pages = static_cast<int>(per_cta);
  }
  if (p.k_chunk_pages < 1) p.k_chunk_pages = 1;

  // Grouped queries (G >= 2, H >= 8) with at most 16 KV heads: the K pass runs
  // on the tensor cores.  A CTA's single producer thread and per-tile chain are
  // serial, so the plan spreads the SM over up to STARKV_KTC_CTAS_PER_SM CTAs,
  // most CTAs first, that fit by registers (the instance's count), shared
  // memory (>= 3 ring stages, 4 for a single CTA) and TMEM (>= 2 accumulators).
  p.ktc = false;
  if (p.log2G >= 1 && p.H >= 8 && p.Hkv <= 16) {
    int log2Hkv = 0;
    while ((1 << log2Hkv) < p.Hkv) ++log2Hkv;
    p.ktc_log2tpt = 7 - log2Hkv;
    p.ktc_ksteps = (p.r + 15) / 16;
    p.ktc_kb = (p.r + 63) / 64;
    p.ktc_nmma = p.H < 16 ? 16 : p.H;
    p.ktc_brows = p.H < 16 ? 32 : 2 * p.H;   // the low-part MMA reads rows [H, H + nmma)
    p.ktc_a_bytes = static_cast<uint32_t>(p.ktc_kb) * 128u * 128u;
    p.ktc_b_bytes = static_cast<uint32_t>(p.ktc_kb) * p.ktc_brows * 128u;
    const int regs = ktc_num_regs(p.log2G, p.H);
    for (int ctas = STARKV_KTC_CTAS_PER_SM; ctas >= 1 && !p.ktc; --ctas) {
      const int per_warp = (regs * 32 + 255) / 256 * 256;
      if (regs <= 0 || per_warp * (kKTCThreads / 32) * ctas * 11 > 65536 * 10) continue;  // 10% margin
      int nacc = 512 / (ctas * p.ktc_nmma);
      if (nacc > kKTCMaxAcc) nacc = kKTCMaxAcc;
      if (nacc < 2) continue;
      // one or two query-tile slots: two hide the reload at a segment boundary, one
      // leaves room for another ring stage (more bytes in flight); a CTA crosses
      // only a few segment boundaries, so the extra stage wins when there is one
      int best_stages = 0, best_nbs = 0;
      uint32_t best_fixed = 0;
      for (int nbs = 2; nbs >= 1; --nbs) {
        // query slots, then full/empty per stage, bfull/bempty[2], tfull/tempty per accumulator, mmadone
        const uint32_t fixed = 1024u + nbs * p.ktc_b_bytes + (4 + 2 * kKTCMaxAcc + 1) * 8u;
        const uint32_t budget = static_cast<uint32_t>(STARKV_KTC_SMEM_BYTES) / ctas - (ctas > 1 ? 1024u : 0u);
        if (budget <= fixed) continue;
        int stages = static_cast<int>((budget - fixed) / (p.ktc_a_bytes + 16u));
        if (stages > 12) stages = 12;
        if (stages > best_stages) { best_stages = stages; best_nbs = nbs; best_fixed = fixed; }
      }
      if (best_stages >= (ctas > 1 ? 3 : 4)) {
        p.ktc = true;
        p.ktc_nacc = nacc; p.ktc_nbs = best_nbs; p.ktc_stages = best_stages;
        p.ktc_tmem = static_cast<uint32_t>(pow2_ceil(nacc * p.ktc_nmma < 32 ? 32 : nacc * p.ktc_nmma));
        p.ktc_smem = best_fixed + static_cast<size_t>(best_stages) * (p.ktc_a_bytes + 16u);
        p.k_ctas = sms * ctas;
      }
    }
  }

  // V pass: R split into ranges of <= 1024 rows (128-row UMMA tiles)
  if (p.R <= STARKV_V_RRANGE) { p.n_rr = 1; p.r_range = p.R; }
  else {
    p.n_rr = (p.R + STARKV_V_RRANGE - 1) / STARKV_V_RRANGE;
    p.r_range = ((p.R + p.n_rr - 1) / p.n_rr + 127) / 128 * 128;
  }
  p.r_range_pad = (p.r_range + 127) / 128 * 128;
  p.n_chunks = p.r_range_pad / 64;
  p.n_mtiles = p.r_range_pad / 128;
  p.vtile = static_cast<uint32_t>(p.r_range_pad) * 16 * 2;
  p.ltile = 16u * p.H * 4;
  p.ptile = static_cast<uint32_t>(p.npad) * 16 * 2;
  p.tmem_cols = static_cast<uint32_t>(pow2_ceil(p.n_mtiles * p.npad < 32 ? 32 : p.n_mtiles * p.npad));
  // pages per ring stage: at most STARKV_V_PPS, fewer while a ring of 3 stages would not fit
  p.v_pps = STARKV_V_PPS < kMaxPPS ? STARKV_V_PPS : kMaxPPS;
  while (p.v_pps > 1 &&
         3u * p.v_pps * (p.vtile + p.ltile + p.ptile) > static_cast<uint32_t>(STARKV_V_RING_BYTES))
    --p.v_pps;
  const uint32_t stage = p.v_pps * (p.vtile + p.ltile + p.ptile);
  p.v_stages = static_cast<int>(static_cast<uint32_t>(STARKV_V_RING_BYTES) / stage);
  if (p.v_stages > 8) p.v_stages = 8;
  if (p.v_stages < 2) p.v_stages = 2;
  p.v_smem = 1024 + static_cast<size_t>(p.v_stages) * stage + p.v_stages * sizeof(StageMeta) +
             (3 * p.v_stages + 4) * sizeof(uint64_t) + (p.npad + 128) * sizeof(float);
  int per_sm = static_cast<int>((227u * 1024u) / (p.v_smem + 1024));
  if (per_sm > static_cast<int>(512 / p.tmem_cols)) per_sm = 512 / p.tmem_cols;
  if (per_sm < 1) per_sm = 1;
  if (per_sm > 2) per_sm = 2;
  p.v_per_sm = per_sm;
  p.v_ctas = sms * per_sm / p.n_rr;
  // a call with few pages gives each CTA at least STARKV_V_MIN_PAGES of them:
  // every CTA boundary inside a sequence costs a Z partial (H x R range fp32)
  // that the finish reads back, which at batch 1 outweighs the pages' codes
  {
    const int64_t pages_max = static_cast<int64_t>(batch) * ((p.cap + 15) / 16);
    const int64_t cap_ctas = (pages_max + STARKV_V_MIN_PAGES - 1) / STARKV_V_MIN_PAGES;
    if (cap_ctas < p.v_ctas) p.v_ctas = static_cast<int>(cap_ctas);
  }
  if (p.v_ctas < 1) p.v_ctas = 1;

  // finish: a stage holds two 64x64 B_V boxes, the hi and lo operand tiles
  // (npad rows x 128 B each) and the partial rows a batch tile can need (its
  // sequences plus one per V-pass CTA boundary, 256 B each); two stages.  The
  // batch tile is the largest (<= 256 sequences, halving) whose stages fit.
  // The epilogue's [npad][128] fp32 sums reuse the ring (two stages hold them).
  p.up_mt = (p.d + 127) / 128;    // 128-row tiles of d (rows past d are ignored)
  p.up_stages = 2;
  p.up_bt_rows = batch < kFinMaxRows ? (batch > 0 ? batch : 1) : kFinMaxRows;
  for (;;) {
    p.up_npad = p.up_bt_rows < 16 ? 16 : (p.up_bt_rows + 15) / 16 * 16;
    const int need = p.up_bt_rows + p.v_ctas - 1;
    p.up_zrows = (need + kFinZBox - 1) / kFinZBox * kFinZBox;
    p.up_stage_bytes = static_cast<uint32_t>(
        align_up(2u * kFinKC * 128u + 2u * static_cast<size_t>(p.up_npad) * 128u + p.up_zrows * 256u, 1024));
    p.up_smem = 1024 + static_cast<size_t>(p.up_stages) * p.up_stage_bytes + (3 * p.up_stages + 1) * sizeof(uint64_t) +
                3 * kFinMaxRows * 4;
    if (p.up_smem <= 220u * 1024u || p.up_bt_rows <= 16) break;
    p.up_bt_rows = p.up_bt_rows / 2 < 16 ? 16 : p.up_bt_rows / 2 / 16 * 16;
  }
  p.up_bt = batch > 0 ? (batch + p.up_bt_rows - 1) / p.up_bt_rows : 1;
  p.up_ks = 1;
  while (p.up_ks < 8 && p.H * p.up_mt * p.up_bt * p.up_ks * 2 <= sms && p.R / kFinKC >= p.up_ks * 2)
    p.up_ks *= 2;
  p.up_kpc = ((p.R + p.up_ks * kFinKC - 1) / (p.up_ks * kFinKC)) * kFinKC;
  p.up_tmem = static_cast<uint32_t>(pow2_ceil(p.up_npad < 32 ? 32 : p.up_npad));

  // workspace layout
  starkv_workspace_layout& w = p.ws;
  size_t off = 0;
  w.status_off = off; off += 256;
  w.prefix_off = off; off = align_up(off + (static_cast<size_t>(batch) + 1) * 4, 256);
  const size_t teff_off = off; off = align_up(off + static_cast<size_t>(batch) * 4, 256);
  (void)teff_off;
  w.qt_off = off; off = align_up(off + static_cast<size_t>(batch) * p.H * p.r * 4, 256);
  w.logits_off = off; off = align_up(off + static_cast<size_t>(batch) * p.t_pad * p.H * 4, 256);
  w.k_ctas = p.k_ctas;
  w.k_slots = batch;   // one maximum per (sequence, head)
  w.mpart_off = off; off = align_up(off + static_cast<size_t>(w.k_slots) * p.H * 4, 256);
  w.v_ctas = p.v_ctas;
  w.v_slots = p.v_ctas + batch;
  w.lpart_off = off; off = align_up(off + static_cast<size_t>(w.v_slots) * p.H * 4, 256);
  w.n_rranges = p.n_rr;
  w.r_range = p.r_range;
  w.zpart_off = off;
  off = align_up(off + static_cast<size_t>(p.n_rr) * w.v_slots * p.H * p.r_range * 4, 256);
  w.k_tensor = p.ktc ? 1 : 0;
  w.qth_off = 0;
  if (p.ktc) { w.qth_off = off; off = align_up(off + static_cast<size_t>(batch) * 2 * p.H * p.r * 2, 256); }
  w.t_pad = p.t_pad;
  w.total_bytes = off;
  return STARKV_OK;
}

// The K pass's page-chunk counter sits in the workspace's status area, 64
// bytes after the status word; the absorption kernel sets it to 0.
constexpr size_t kWorkCtrOffset = 64;

size_t teff_offset(const DecodePlan& p) {
  return align_up(p.ws.prefix_off + (static_cast<size_t>(p.B) + 1) * 4, 256);
}

// ------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    else
      cudaGetLastError();
  });
  return fn;
}

// Row-major fp16 matrix [rows][cols] as a 2-D tensor map with boxes of
// box_cols (x 2 bytes = 128 bytes) by box_rows and the 128-byte swizzle.
bool encode_2d_map(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                   uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Row-major fp32 matrix [rows][cols] as a 2-D tensor map with boxes of
// box_cols x box_rows, no swizzle (rows land back to back in shared memory).
bool encode_f32_rows_map(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                         uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// V pool [num_blocks*16 tokens][R] fp16 as a 3-D tensor map {64 codes, tokens,
// R/64 column blocks} (strides: a token row, then 128 bytes per block) with
// boxes {64, 16 tokens, box_chunks}: one copy brings a page's R range as
// box_chunks consecutive 64-code x 16-token blocks of 2 KiB, each already the
// 128B-swizzled MN-major operand slice; blocks past R read as zero.
bool encode_vpool_map(CUtensorMap* map, const void* v_cache, int R, int NB, uint32_t box_chunks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(NB) * 16, static_cast<cuuint64_t>(R) / 64};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(R) * 2, 128};
  cuuint32_t box[3] = {64, 16, box_chunks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult res = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(v_cache), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

// K pool [num_blocks*16 tokens][Hkv][r] fp16 as a 3-D tensor map {r, Hkv,
// tokens} with boxes {64 codes, box_heads heads, box_tokens} and the 128-byte
// swizzle (codes past r read as zero).
bool encode_kpool_map(CUtensorMap* map, const void* k_cache, int r, int Hkv, int NB, uint32_t box_heads,
                      uint32_t box_tokens) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(r), static_cast<cuuint64_t>(Hkv),
                        static_cast<cuuint64_t>(NB) * 16};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(r) * 2, static_cast<cuuint64_t>(Hkv) * r * 2};
  cuuint32_t box[3] = {64, box_heads, box_tokens};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult res = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(k_cache), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

// Every kernel is launched with programmatic stream serialisation: the grid may
// start while the previous grid in the stream drains, and waits for it inside
// (griddep_wait) before touching memory.  cluster_y > 1 adds a (1, cluster_y, 1)
// thread-block cluster.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster_y,
                   Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_y > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 1;
    attr[n].val.clusterDim.y = static_cast<unsigned>(cluster_y);
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) cudaGetLastError();
  return e;
}

template <int G, int H>
cudaError_t launch_kpass_tc_gh(const DecodePlan& pl, const CUtensorMap& kmap, const CUtensorMap& qmap,
                               const KPassTCParams& tp, cudaStream_t s) {
  if (!set_smem(kpass_tc_kernel<G, H>, pl.ktc_smem)) return cudaErrorInvalidValue;
  return launch(kpass_tc_kernel<G, H>, dim3(pl.k_ctas), dim3(kKTCThreads), pl.ktc_smem, s, 1, kmap, qmap, tp);
}

template <int H>
cudaError_t launch_kpass_tc_h(const DecodePlan& pl, const CUtensorMap& kmap, const CUtensorMap& qmap,
                              const KPassTCParams& tp, cudaStream_t s) {
  // G = H / Hkv with 1 <= Hkv <= 16 and G >= 2
  switch (pl.log2G) {
    case 1: if constexpr (H / 2 <= 16) return launch_kpass_tc_gh<2, H>(pl, kmap, qmap, tp, s); break;
    case 2: if constexpr (H >= 4) return launch_kpass_tc_gh<(H >= 4 ? 4 : H), H>(pl, kmap, qmap, tp, s); break;
    case 3: if constexpr (H >= 8) return launch_kpass_tc_gh<(H >= 8 ? 8 : H), H>(pl, kmap, qmap, tp, s); break;
    case 4: if constexpr (H >= 16) return launch_kpass_tc_gh<(H >= 16 ? 16 : H), H>(pl, kmap, qmap, tp, s); break;
    case 5: if constexpr (H >= 32) return launch_kpass_tc_gh<(H >= 32 ? 32 : H), H>(pl, kmap, qmap, tp, s); break;
    case 6: if constexpr (H >= 64) return launch_kpass_tc_gh<(H >= 64 ? 64 : H), H>(pl, kmap, qmap, tp, s); break;
    default: break;
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_kpass_tc(const DecodePlan& pl, const CUtensorMap& kmap, const CUtensorMap& qmap,
                            const KPassTCParams& tp, cudaStream_t s) {
  switch (pl.H) {
    case 8: return launch_kpass_tc_h<8>(pl, kmap, qmap, tp, s);
    case 16: return launch_kpass_tc_h<16>(pl, kmap, qmap, tp, s);
    case 32: return launch_kpass_tc_h<32>(pl, kmap, qmap, tp, s);
    default: return launch_kpass_tc_h<64>(pl, kmap, qmap, tp, s);
  }
}

template <int L, int CPT>
cudaError_t launch_kpass(const DecodePlan& pl, const KPassParams& kp, cudaStream_t s) {
  if (!set_smem(kpass_kernel<L, CPT>, pl.k_smem)) return cudaErrorInvalidValue;
  return launch(kpass_kernel<L, CPT>, dim3(pl.k_ctas), dim3(kKThreads), pl.k_smem, s, 1, kp);
}

}  // namespace
}  // namespace starkv

using namespace starkv;

extern "C" {

const char* starkv_status_string(starkv_status s) {
  switch (s) {
    case STARKV_OK: return "STARKV_OK";
    case STARKV_ERR_INVALID_ARG: return "STARKV_ERR_INVALID_ARG";
    case STARKV_ERR_UNSUPPORTED: return "STARKV_ERR_UNSUPPORTED";
    case STARKV_ERR_WORKSPACE: return "STARKV_ERR_WORKSPACE";
    case STARKV_ERR_CUDA: return "STARKV_ERR_CUDA";
    case STARKV_ERR_DEVICE_CHECK: return "STARKV_ERR_DEVICE_CHECK";
    case STARKV_ERR_TIMEOUT: return "STARKV_ERR_TIMEOUT";
  }
  return "STARKV_UNKNOWN_STATUS";
}

int32_t starkv_version(void) { return 200; }

int64_t starkv_kv_bytes_per_token(int32_t n_layers, const int32_t* num_heads, const int32_t* k_ranks,
                                  const int32_t* v_ranks) {
  if (n_layers <= 0 || !num_heads || !k_ranks || !v_ranks) return -1;
  int64_t codes = 0;
  for (int32_t l = 0; l < n_layers; ++l) {
    if (num_heads[l] <= 0 || k_ranks[l] <= 0 || v_ranks[l] <= 0) return -1;
    codes += static_cast<int64_t>(num_heads[l]) * k_ranks[l] + v_ranks[l];
  }
  return 2 * codes;
}

int64_t starkv_num_blocks(int64_t budget_bytes, int64_t bytes_per_token, int32_t block_size) {
  if (budget_bytes < 0 || bytes_per_token <= 0 || block_size <= 0) return -1;
  return budget_bytes / (static_cast<int64_t>(block_size) * bytes_per_token);
}

int32_t starkv_rank_from_spectrum(const double* s, int32_t n, double tau) {
  if (n < 0 || (n > 0 && !s) || std::isnan(tau)) return -1;
  int32_t c = 0;
  for (int32_t i = 0; i < n; ++i)
    if (s[i] > tau) ++c;
  return c;
}

namespace {
// Launch plan of the append roles of the prep kernel: the V-code GEMM tiles
// and the K-code items of `batch` new rows of k, v stored at `tgt`.
struct AppendPlan {
  CUtensorMap amap, vmap;
  AppendVParams vp{};
  AppendKParams kp{};
  int v_mt, v_cols, KS;
  size_t v_smem, k_smem;
};

starkv_status plan_append(const starkv_layer_desc* desc, int32_t batch, const void* k, const void* v,
                          const void* A_K, const void* A_V, AppendTarget tgt, void* k_cache, void* v_cache,
                          AppendPlan* ap) {
  if (!k || !v || !A_K || !A_V || !k_cache || !v_cache) return STARKV_ERR_INVALID_ARG;
  if (!tgt.slots && (!tgt.tables || !tgt.positions)) return STARKV_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(A_K) || !aligned16(A_V) || !aligned16(k_cache) ||
      !aligned16(v_cache) || (reinterpret_cast<uintptr_t>(tgt.tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(tgt.positions) & 3u) || (reinterpret_cast<uintptr_t>(tgt.slots) & 3u))
    return STARKV_ERR_INVALID_ARG;
  const int H = kv_heads(desc), d = desc->head_dim, r = desc->k_rank, R = desc->v_rank;   // codes per KV head
  const int HD = H * d;
  // joint V codes: tcgen05 GEMM, split-K over a cluster
  const int n_bt = (batch + 255) / 256;
  const int bt_rows = batch < 256 ? batch : 256;
  const int npad = (bt_rows + 15) / 16 * 16;
  if (!encode_2d_map(&ap->amap, A_V, static_cast<uint64_t>(R), static_cast<uint64_t>(HD), 64, kAppKC) ||
      !encode_2d_map(&ap->vmap, v, static_cast<uint64_t>(HD), static_cast<uint64_t>(batch), 64,
                     static_cast<uint32_t>(npad)))
    return STARKV_ERR_CUDA;
  ap->v_mt = (R + 127) / 128;
  ap->v_cols = ap->v_mt * n_bt;
  const int sms = device_sm_count();
  int KS = 1;
  // <= one wave at 2 CTAs/SM, and clusters of at most 4: the whole prep grid
  // (K-code and absorption items too) is launched in clusters of KS, and with
  // 8 some of them found no free GPC slots until the V tiles had ended
  while (KS < STARKV_APP_KS_MAX && ap->v_cols * KS * 2 <= 2 * sms && (HD / kAppKC) >= KS * 2) KS *= 2;
  ap->KS = KS;
  AppendVParams& vp = ap->vp;
  vp.tgt = tgt;
  vp.v_cache = static_cast<__half*>(v_cache);
  vp.B = batch; vp.HD = HD; vp.R = R;
  vp.k_per_cta = ((HD + KS * kAppKC - 1) / (KS * kAppKC)) * kAppKC;
  vp.npad = npad;
  vp.stages = 4;
  vp.tmem_cols = static_cast<uint32_t>(pow2_ceil(npad < 32 ? 32 : npad));
  const size_t stage_bytes = 2u * kAppKC * 128u + static_cast<size_t>(npad) * 128u;
  ap->v_smem = vp.stages * stage_bytes + (2 * vp.stages + 1) * sizeof(uint64_t);
  // head-wise K codes
  AppendKParams& kp = ap->kp;
  kp.tgt = tgt;
  kp.k = static_cast<const __half*>(k);
  kp.A_K = static_cast<const __half*>(A_K);
  kp.k_cache = static_cast<__half*>(k_cache);
  kp.H = H; kp.d = d; kp.r = r;
  kp.B = batch;
  kp.tile = kAppKB;
  ap->k_smem = (static_cast<size_t>(d) * r + static_cast<size_t>(kAppKB) * d) * 2;
  return STARKV_OK;
}

// One prep launch: the append roles of `app` (null: none) and the query
// absorption `abs` (null: none) over `batch` rows.  Item tiles of 16 rows are
// used when they keep the grid within one wave of two CTAs per SM, else 32.
starkv_status launch_prep(int d, const AppendPlan* app, const AbsorbParams* abs, int batch, cudaStream_t s) {
  PrepParams pp{};
  std::memset(&pp, 0, sizeof(pp));
  const int KS = app ? app->KS : 1;
  const int sms = device_sm_count();
  const int v_ctas = app ? app->v_cols * KS : 0;
  const int spare = 2 * sms - v_ctas > 2 * KS ? 2 * sms - v_ctas : 2 * KS;
  const int k_heads = app ? app->kp.H : 0;
  const int a_heads = abs ? abs->H : 0;
  const int r = app ? app->kp.r : abs->r;
  int tile = 16;
  if ((k_heads + a_heads) * ((batch + tile - 1) / tile) > spare) tile = kAbsBT;
  // an absorption alone over many rows (a chunked prefill): items of 128 rows,
  // so that each B_K slice is staged for 4x more rows and the grid stays
  // within a few waves
  if (!app && a_heads * ((batch + tile - 1) / tile) > 2 * spare) tile = kAbsBigTile;
  size_t smem = 0;
  CUtensorMap none;
  std::memset(&none, 0, sizeof(none));
  if (app) {
    pp.v = app->vp;
    pp.k = app->kp;
    pp.k.tile = tile;
    pp.v_mt = app->v_mt;
    pp.v_cols = app->v_cols;
    pp.k_items = k_heads * ((batch + tile - 1) / tile);
    pp.k_cols = (pp.k_items + KS - 1) / KS;
    smem = app->v_smem > app->k_smem ? app->v_smem : app->k_smem;
  }
  if (abs) {
    pp.a = *abs;
    pp.a_tile = tile;
    pp.a_items = a_heads * ((batch + tile - 1) / tile);
    const size_t ws = (static_cast<size_t>(d) * r + static_cast<size_t>(tile) * d) * 2;   // B_K^T + q rows
    if (ws > smem) smem = ws;
  }
  smem += 1024;   // room to align the dynamic shared memory to 1024 bytes
  const dim3 grid(pp.v_cols + pp.k_cols + (pp.a_items + KS - 1) / KS, KS);
  const CUtensorMap& amap = app ? app->amap : none;
  const CUtensorMap& vmap = app ? app->vmap : none;
  if (!set_smem(prep_kernel, smem)) return STARKV_ERR_CUDA;
  return launch(prep_kernel, grid, dim3(kPrepThreads), smem, s, KS, amap, vmap, pp) == cudaSuccess ? STARKV_OK
                                                                                                   : STARKV_ERR_CUDA;
}

// Compress rows of k, v and store their codes at the target rows (see AppendTarget).
starkv_status compress_store_impl(const starkv_layer_desc* desc, int32_t batch, const void* k, const void* v,
                                  const void* A_K, const void* A_V, AppendTarget tgt, void* k_cache,
                                  void* v_cache, void* stream) {
  starkv_status st = check_desc(desc);
  if (st != STARKV_OK) return st;
  if (batch < 0) return STARKV_ERR_INVALID_ARG;
  if (batch == 0) return STARKV_OK;
  AppendPlan ap{};
  st = plan_append(desc, batch, k, v, A_K, A_V, tgt, k_cache, v_cache, &ap);
  if (st != STARKV_OK) return st;
  return launch_prep(desc->head_dim, &ap, nullptr, batch, static_cast<cudaStream_t>(stream));
}
}  // namespace

starkv_status starkv_compress_append(const starkv_layer_desc* desc, int32_t batch, const void* k, const void* v,
                                     const void* A_K, const void* A_V, const int32_t* block_tables,
                                     const int32_t* positions, void* k_cache, void* v_cache, int32_t* status,
                                     void* stream) {
  if (batch > 0 && (!block_tables || !positions)) return STARKV_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(status) & 3u) return STARKV_ERR_INVALID_ARG;
  AppendTarget tgt{nullptr, block_tables, positions, desc ? desc->max_blocks_per_seq : 0,
                   desc ? desc->num_blocks : 0, status};
  return compress_store_impl(desc, batch, k, v, A_K, A_V, tgt, k_cache, v_cache, stream);
}

starkv_status starkv_compress_store(const starkv_layer_desc* desc, int32_t n_tokens, const void* k, const void* v,
                                    const void* A_K, const void* A_V, const int32_t* slot_mapping, void* k_cache,
                                    void* v_cache, int32_t* status, void* stream) {
  if (n_tokens > 0 && !slot_mapping) return STARKV_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(status) & 3u) return STARKV_ERR_INVALID_ARG;
  AppendTarget tgt{slot_mapping, nullptr, nullptr, desc ? desc->max_blocks_per_seq : 0,
                   desc ? desc->num_blocks : 0, status};
  return compress_store_impl(desc, n_tokens, k, v, A_K, A_V, tgt, k_cache, v_cache, stream);
}

// Test hook state: the dropped K-pass stage applies to every later decode.
namespace {
std::atomic<int> g_drop_k_stage{-1};
}

starkv_status starkv_set_wait_test_hook(uint32_t wait_limit_us, int32_t drop_k_stage) {
  if (drop_k_stage < -1) return STARKV_ERR_INVALID_ARG;
  const uint64_t ns = wait_limit_us ? static_cast<uint64_t>(wait_limit_us) * 1000ull : kWaitLimitNs;
  if (cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns)) != cudaSuccess) {
    cudaGetLastError();
    return STARKV_ERR_CUDA;
  }
  g_drop_k_stage.store(drop_k_stage);
  return STARKV_OK;
}

size_t starkv_decode_workspace_bytes(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len) {
  DecodePlan pl{};
  if (make_plan(desc, batch, max_seq_len, &pl) != STARKV_OK) return 0;
  return pl.ws.total_bytes;
}

starkv_status starkv_decode_workspace_layout(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len,
                                             starkv_workspace_layout* out) {
  if (!out) return STARKV_ERR_INVALID_ARG;
  DecodePlan pl{};
  starkv_status st = make_plan(desc, batch, max_seq_len, &pl);
  if (st != STARKV_OK) return st;
  *out = pl.ws;
  return STARKV_OK;
}

namespace {
// A call with nothing to compute still leaves a clean status word in the
// workspace it was given, so that starkv_decode_check() after any successful
// call reads this call's status and not stale bytes.
starkv_status clear_status(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < sizeof(int32_t)) return STARKV_OK;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u)) return STARKV_ERR_WORKSPACE;
  if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return STARKV_ERR_CUDA;
  }
  return STARKV_OK;
}

starkv_status decode_impl(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len, const void* q,
                          const void* B_K, const void* B_V, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* seq_lens, float scale, void* workspace,
                          size_t workspace_bytes, void* out, void* stream, void* const* stage_events,
                          const int32_t* row_seq = nullptr, const AppendPlan* app = nullptr) {
  DecodePlan pl{};
  starkv_status st = make_plan(desc, batch, max_seq_len, &pl);
  if (st != STARKV_OK) return st;
  if (!(std::isfinite(scale) && scale > 0.f)) return STARKV_ERR_INVALID_ARG;
  if (batch == 0) return clear_status(workspace, workspace_bytes, stream);
  if (!q || !B_K || !B_V || !k_cache || !v_cache || !block_tables || !seq_lens || !out)
    return STARKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(B_K) || !aligned16(B_V) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return STARKV_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.ws.total_bytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return STARKV_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(ws + pl.ws.status_off);
  int32_t* prefix = reinterpret_cast<int32_t*>(ws + pl.ws.prefix_off);
  int32_t* teff = reinterpret_cast<int32_t*>(ws + teff_offset(pl));
  float* qt = reinterpret_cast<float*>(ws + pl.ws.qt_off);
  float* logits = reinterpret_cast<float*>(ws + pl.ws.logits_off);
  float* mpart = reinterpret_cast<float*>(ws + pl.ws.mpart_off);
  float* lpart = reinterpret_cast<float*>(ws + pl.ws.lpart_off);
  float* zpart = reinterpret_cast<float*>(ws + pl.ws.zpart_off);
  uint32_t* work_ctr = reinterpret_cast<uint32_t*>(ws + pl.ws.status_off + kWorkCtrOffset);

  if (max_seq_len == 0) {
    if (app && launch_prep(pl.d, app, nullptr, batch, s) != STARKV_OK) return STARKV_ERR_CUDA;
    if (cudaMemsetAsync(status, 0, 4, s) != cudaSuccess ||
        cudaMemsetAsync(out, 0, static_cast<size_t>(batch) * pl.H * pl.d * 2, s) != cudaSuccess)
      return STARKV_ERR_CUDA;
    return STARKV_OK;
  }

  CUtensorMap vmap, bvmap, zmap;
  if (!encode_vpool_map(&vmap, v_cache, pl.R, pl.NB, static_cast<uint32_t>(pl.n_chunks))) return STARKV_ERR_CUDA;
  if (!encode_2d_map(&bvmap, B_V, static_cast<uint64_t>(pl.Hkv) * pl.d, static_cast<uint64_t>(pl.R), 64, kFinKC) ||
      !encode_f32_rows_map(&zmap, zpart, static_cast<uint64_t>(pl.r_range),
                           static_cast<uint64_t>(pl.n_rr) * pl.H * pl.ws.v_slots, 64, kFinZBox))
    return STARKV_ERR_CUDA;
  auto mark = [&](int i) {
    if (stage_events && stage_events[i]) cudaEventRecord(static_cast<cudaEvent_t>(stage_events[i]), s);
  };
  mark(0);

  AbsorbParams ap{};
  ap.q = static_cast<const __half*>(q);
  ap.B_K = static_cast<const __half*>(B_K);
  ap.seq_lens = seq_lens;
  ap.qt = qt; ap.prefix = prefix; ap.teff = teff; ap.status = status;
  __half* qth = pl.ktc ? reinterpret_cast<__half*>(ws + pl.ws.qth_off) : nullptr;
  ap.qth = qth;
  ap.mpart_init = mpart;   // both K passes merge each sequence's maxima by float-max atomics
  ap.n_mpart = pl.ws.k_slots * pl.H;
  ap.work_ctr = work_ctr;
  ap.B = batch; ap.H = pl.H; ap.d = pl.d; ap.r = pl.r; ap.cap = pl.cap; ap.log2G = pl.log2G;
  ap.coef = scale * kLog2e;
  // the query absorption, with the step's compress-and-append in the same launch when fused
  if (launch_prep(pl.d, app, &ap, batch, s) != STARKV_OK) return STARKV_ERR_CUDA;
  mark(1);

  KPassParams kp{};
  kp.k_cache = static_cast<const __half*>(k_cache);
  kp.tables = block_tables; kp.row_seq = row_seq; kp.teff = teff; kp.prefix = prefix; kp.qt = qt;
  kp.logits = logits; kp.mpart = mpart; kp.status = status;
  kp.work_ctr = work_ctr; kp.chunk_pages = pl.k_chunk_pages;
  kp.B = batch; kp.H = pl.H; kp.log2H = pl.log2H; kp.r = pl.r; kp.MB = pl.MB; kp.NB = pl.NB; kp.t_pad = pl.t_pad;
  kp.Hkv = pl.Hkv; kp.log2G = pl.log2G;
  kp.tps = pl.tps; kp.stages = pl.k_stages; kp.stage_bytes = pl.k_stage_bytes;
  kp.drop_stage = g_drop_k_stage.load(std::memory_order_relaxed);
  cudaError_t e;
  if (pl.ktc) {
    CUtensorMap kmap, qmap;
    const uint32_t tpt = 1u << pl.ktc_log2tpt;
    if (!encode_kpool_map(&kmap, k_cache, pl.r, pl.Hkv, pl.NB, static_cast<uint32_t>(pl.Hkv), tpt < 16 ? tpt : 16) ||
        !encode_2d_map(&qmap, qth, static_cast<uint64_t>(pl.r), static_cast<uint64_t>(batch) * 2 * pl.H, 64,
                       static_cast<uint32_t>(pl.ktc_brows)))
      return STARKV_ERR_CUDA;
    KPassTCParams tp{};
    tp.tables = block_tables; tp.row_seq = row_seq; tp.teff = teff; tp.prefix = prefix;
    tp.logits = logits; tp.mpart = mpart; tp.status = status;
    tp.B = batch; tp.log2G = pl.log2G; tp.log2Hkv = pl.log2H - pl.log2G;
    tp.MB = pl.MB; tp.NB = pl.NB; tp.t_pad = pl.t_pad;
    tp.log2tpt = pl.ktc_log2tpt; tp.ksteps = pl.ktc_ksteps; tp.kb = pl.ktc_kb;
    tp.nmma = pl.ktc_nmma; tp.brows = pl.ktc_brows;
    tp.nacc = pl.ktc_nacc; tp.nbs = pl.ktc_nbs; tp.stages = pl.ktc_stages;
    tp.a_bytes = pl.ktc_a_bytes; tp.b_bytes = pl.ktc_b_bytes; tp.tmem_cols = pl.ktc_tmem;
    tp.drop_stage = kp.drop_stage;
    e = launch_kpass_tc(pl, kmap, qmap, tp, s);
  } else if (pl.L == 1 && pl.CPT == 4) e = launch_kpass<1, 4>(pl, kp, s);
  else if (pl.L == 1 && pl.CPT == 8) e = launch_kpass<1, 8>(pl, kp, s);
  else if (pl.L == 1) e = launch_kpass<1, 12>(pl, kp, s);
  else if (pl.L == 2) e = launch_kpass<2, 8>(pl, kp, s);
  else e = launch_kpass<4, 8>(pl, kp, s);
  if (e != cudaSuccess) return STARKV_ERR_CUDA;
  mark(2);

  VPassParams vp{};
  vp.tables = block_tables; vp.row_seq = row_seq; vp.teff = teff; vp.prefix = prefix; vp.logits = logits;
  vp.mpart = mpart;
  vp.zpart = zpart; vp.lpart = lpart; vp.status = status;
  vp.B = batch; vp.H = pl.H; vp.npad = pl.npad; vp.MB = pl.MB; vp.NB = pl.NB; vp.R = pl.R;
  vp.t_pad = pl.t_pad; vp.r_range = pl.r_range; vp.n_rr = pl.n_rr; vp.v_slots = pl.ws.v_slots;
  vp.stages = pl.v_stages; vp.n_chunks = pl.n_chunks; vp.n_mtiles = pl.n_mtiles; vp.tmem_cols = pl.tmem_cols;
  vp.vtile_bytes = pl.vtile; vp.ltile_bytes = pl.ltile; vp.ptile_bytes = pl.ptile; vp.pps = pl.v_pps;
  if (!set_smem(vpass_kernel<false>, pl.v_smem)) return STARKV_ERR_CUDA;
  if (launch(vpass_kernel<false>, dim3(pl.v_ctas, pl.n_rr), dim3(kVThreads), pl.v_smem, s, 1, vmap, vp) != cudaSuccess)
    return STARKV_ERR_CUDA;
  mark(3);

  FinishParams fp{};
  fp.out = static_cast<__half*>(out);
  fp.zpart = zpart; fp.lpart = lpart; fp.prefix = prefix;
  fp.B = batch; fp.H = pl.H; fp.d = pl.d; fp.R = pl.R; fp.log2G = pl.log2G;
  fp.r_range = pl.r_range; fp.v_slots = pl.ws.v_slots; fp.v_grid = pl.v_ctas;
  fp.n_mt = pl.up_mt; fp.bt_rows = pl.up_bt_rows; fp.k_per_cta = pl.up_kpc; fp.npad = pl.up_npad;
  fp.stages = pl.up_stages; fp.zrows = pl.up_zrows; fp.stage_bytes = pl.up_stage_bytes; fp.tmem_cols = pl.up_tmem;
  if (!set_smem(finish_kernel, pl.up_smem)) return STARKV_ERR_CUDA;
  if (launch(finish_kernel, dim3(pl.H * pl.up_mt * pl.up_bt, pl.up_ks), dim3(kFinThreads), pl.up_smem, s, pl.up_ks,
             bvmap, zmap, fp) != cudaSuccess)
    return STARKV_ERR_CUDA;
  mark(4);
  return STARKV_OK;
}
}  // namespace

starkv_status starkv_paged_decode(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len,
                                  const void* q, const void* B_K, const void* B_V, const void* k_cache,
                                  const void* v_cache, const int32_t* block_tables, const int32_t* seq_lens,
                                  float scale, void* workspace, size_t workspace_bytes, void* out, void* stream) {
  return decode_impl(desc, batch, max_seq_len, q, B_K, B_V, k_cache, v_cache, block_tables, seq_lens, scale,
                     workspace, workspace_bytes, out, stream, nullptr);
}

starkv_status starkv_append_decode(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len,
                                   const void* k, const void* v, const void* A_K, const void* A_V,
                                   const int32_t* positions, const void* q, const void* B_K, const void* B_V,
                                   void* k_cache, void* v_cache, const int32_t* block_tables,
                                   const int32_t* seq_lens, float scale, void* workspace, size_t workspace_bytes,
                                   void* out, int32_t* append_status, void* stream) {
  starkv_status st = check_desc(desc);
  if (st != STARKV_OK) return st;
  if (batch < 0) return STARKV_ERR_INVALID_ARG;
  if (batch == 0) return clear_status(workspace, workspace_bytes, stream);
  if (!block_tables || !positions || (reinterpret_cast<uintptr_t>(append_status) & 3u)) return STARKV_ERR_INVALID_ARG;
  AppendTarget tgt{nullptr, block_tables, positions, desc->max_blocks_per_seq, desc->num_blocks, append_status};
  AppendPlan ap{};
  st = plan_append(desc, batch, k, v, A_K, A_V, tgt, k_cache, v_cache, &ap);
  if (st != STARKV_OK) return st;
  return decode_impl(desc, batch, max_seq_len, q, B_K, B_V, k_cache, v_cache, block_tables, seq_lens, scale,
                     workspace, workspace_bytes, out, stream, nullptr, nullptr, &ap);
}

// Staging layout of starkv_append_decode_host: the step's inputs and output
// as device copies, each 256-byte aligned.
struct HostStaging {
  size_t k, v, q, pos, lens, tables, out, total;
};

bool host_staging(const starkv_layer_desc* desc, int32_t batch, HostStaging* st) {
  if (check_desc(desc) != STARKV_OK || batch < 0) return false;
  const size_t B = static_cast<size_t>(batch);
  const size_t kv = B * kv_heads(desc) * desc->head_dim * 2, qo = B * desc->num_heads * desc->head_dim * 2;
  size_t off = 0;
  st->k = off; off = align_up(off + kv, 256);
  st->v = off; off = align_up(off + kv, 256);
  st->q = off; off = align_up(off + qo, 256);
  st->pos = off; off = align_up(off + B * 4, 256);
  st->lens = off; off = align_up(off + B * 4, 256);
  st->tables = off; off = align_up(off + B * desc->max_blocks_per_seq * 4, 256);
  st->out = off; off = align_up(off + qo, 256);
  st->total = off > 256 ? off : 256;
  return true;
}

size_t starkv_host_staging_bytes(const starkv_layer_desc* desc, int32_t batch) {
  HostStaging st;
  return host_staging(desc, batch, &st) ? st.total : 0;
}

starkv_status starkv_append_decode_host(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len,
                                        const void* k_host, const void* v_host, const int32_t* positions_host,
                                        const void* q_host, const int32_t* block_tables_host,
                                        const int32_t* seq_lens_host, const void* A_K, const void* A_V,
                                        const void* B_K, const void* B_V, void* k_cache, void* v_cache,
                                        float scale, void* staging, size_t staging_bytes, void* workspace,
                                        size_t workspace_bytes, void* out_host, int32_t* append_status,
                                        void* stream) {
  HostStaging st;
  if (!host_staging(desc, batch, &st)) return check_desc(desc) != STARKV_OK ? check_desc(desc) : STARKV_ERR_INVALID_ARG;
  if (batch == 0) return clear_status(workspace, workspace_bytes, stream);
  if (!k_host || !v_host || !positions_host || !q_host || !block_tables_host || !seq_lens_host || !out_host)
    return STARKV_ERR_INVALID_ARG;
  if (!staging || staging_bytes < st.total || (reinterpret_cast<uintptr_t>(staging) & 255u))
    return STARKV_ERR_WORKSPACE;
  // the decode's own argument checks run before any copy is enqueued
  DecodePlan pl{};
  starkv_status ps = make_plan(desc, batch, max_seq_len, &pl);
  if (ps != STARKV_OK) return ps;
  if (!(std::isfinite(scale) && scale > 0.f)) return STARKV_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < pl.ws.total_bytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return STARKV_ERR_WORKSPACE;
  if (!A_K || !A_V || !B_K || !B_V || !k_cache || !v_cache || !aligned16(A_K) || !aligned16(A_V) ||
      !aligned16(B_K) || !aligned16(B_V) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(append_status) & 3u))
    return STARKV_ERR_INVALID_ARG;
  uint8_t* sg = static_cast<uint8_t*>(staging);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t B = static_cast<size_t>(batch);
  const size_t kv = B * kv_heads(desc) * desc->head_dim * 2, qo = B * desc->num_heads * desc->head_dim * 2;
  // one copy per input (no batched-copy call)
  const struct { size_t off; const void* src; size_t bytes; } in[] = {
      {st.k, k_host, kv}, {st.v, v_host, kv}, {st.q, q_host, qo}, {st.pos, positions_host, B * 4},
      {st.lens, seq_lens_host, B * 4}, {st.tables, block_tables_host, B * desc->max_blocks_per_seq * 4}};
  for (const auto& c : in)
    if (cudaMemcpyAsync(sg + c.off, c.src, c.bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
      cudaGetLastError();
      return STARKV_ERR_CUDA;
    }
  const starkv_status ds = starkv_append_decode(
      desc, batch, max_seq_len, sg + st.k, sg + st.v, A_K, A_V, reinterpret_cast<const int32_t*>(sg + st.pos),
      sg + st.q, B_K, B_V, k_cache, v_cache, reinterpret_cast<const int32_t*>(sg + st.tables),
      reinterpret_cast<const int32_t*>(sg + st.lens), scale, workspace, workspace_bytes, sg + st.out,
      append_status, stream);
  if (ds != STARKV_OK) return ds;
  if (cudaMemcpyAsync(out_host, sg + st.out, qo, cudaMemcpyDeviceToHost, s) != cudaSuccess) {
    cudaGetLastError();
    return STARKV_ERR_CUDA;
  }
  return STARKV_OK;
}

// Prefill workspace: the decode workspace of n_rows rows, then the rows'
// sequence map and lengths (int32 [n_rows] each).
size_t prefill_rows_offset(const DecodePlan& pl) { return align_up(pl.ws.total_bytes, 256); }

namespace {
// ------------------------------------------------- read-once chunked prefill
// A chunk's rows are taken nq = 16 / G at a time as virtual sequences whose
// query heads are the virtual heads (h, i); every K and V page of a virtual
// sequence is then streamed once for all of its rows (see kpass_chunk_kernel).
// Shapes: KV heads in groups of 8 (Hkv % 8 == 0), G = H / Hkv <= 16.
struct ChunkPlan {
  int H, Hkv, d, r, R, G, nq, log2nq, Hv, lw, n_vg, nv_max, n_groups, t_pad, MB, NB, n_rows, n_seqs, n_pc;
  int vpk, kvt, kcols;   // virtual heads per KV head, KV heads per K tile, its UMMA N
  // K pass
  int k_ctas, kb, ksteps, k_stages, nacc, nbs;
  uint32_t a_bytes, b_bytes, k_tmem;
  size_t k_smem;
  // V pass
  int r_range, r_range_pad, n_rr, n_chunks, n_mtiles, v_ctas, v_stages, v_slots, k_slots, v_pps;
  uint32_t vtile, ltile, ptile, v_tmem;
  size_t v_smem;
  // finish
  int up_mt, up_bt_rows, up_bt, up_npad, up_ks, up_kpc, up_zrows;
  uint32_t up_stage_bytes, up_tmem;
  size_t up_smem;
  // workspace
  size_t status_off, prefix_off, teff_off, vs_seq_off, vs_row0_off, vs_nrows_off, vs_len_off, qth_off, logits_off,
      mpart_off, lpart_off, lwpart_off, wts_off, zpart_off, total;
};

cudaError_t launch_kpass_chunk(int vpk, size_t smem, int ctas, const CUtensorMap& kmap, const CUtensorMap& qmap,
                               const KPassChunkParams& kp, cudaStream_t s) {
  if (vpk == 16) {
    if (!set_smem(kpass_chunk_kernel<16>, smem)) return cudaErrorInvalidValue;
    return launch(kpass_chunk_kernel<16>, dim3(ctas), dim3(kKTCThreads), smem, s, 1, kmap, qmap, kp);
  }
  if (vpk == 32) {
    if (!set_smem(kpass_chunk_kernel<32>, smem)) return cudaErrorInvalidValue;
    return launch(kpass_chunk_kernel<32>, dim3(ctas), dim3(kKTCThreads), smem, s, 1, kmap, qmap, kp);
  }
  if (!set_smem(kpass_chunk_kernel<64>, smem)) return cudaErrorInvalidValue;
  return launch(kpass_chunk_kernel<64>, dim3(ctas), dim3(kKTCThreads), smem, s, 1, kmap, qmap, kp);
}

bool chunk_eligible(const starkv_layer_desc* d) {
  const int Hkv = kv_heads(d);
  return Hkv % 8 == 0 && d->num_heads / Hkv <= 16;
}

starkv_status make_chunk_plan(const starkv_layer_desc* d, int32_t n_seqs, int32_t n_rows, int32_t max_seq_len,
                              ChunkPlan* cp) {
  starkv_status st = check_desc(d);
  if (st != STARKV_OK) return st;
  if (n_seqs < 0 || n_rows < 0 || max_seq_len < 0) return STARKV_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_seq_len) > static_cast<int64_t>(d->max_blocks_per_seq) * 16)
    return STARKV_ERR_INVALID_ARG;
  if (!chunk_eligible(d)) return STARKV_ERR_UNSUPPORTED;
  ChunkPlan& c = *cp;
  std::memset(&c, 0, sizeof(c));
  c.H = d->num_heads; c.Hkv = kv_heads(d); c.d = d->head_dim; c.r = d->k_rank; c.R = d->v_rank;
  // VPK virtual heads per KV head: all 16 rows of a chunk (one virtual
  // sequence, pages read once) while G <= 4, 64 of them above (nq = 64 / G)
  c.G = c.H / c.Hkv;
  c.vpk = 16 * c.G < 64 ? 16 * c.G : 64;
  c.nq = c.vpk / c.G;
  c.kvt = c.vpk >= 64 ? 4 : 8;
  c.kcols = c.kvt * c.vpk;
  while ((1 << c.log2nq) < c.nq) ++c.log2nq;
  c.Hv = c.H * c.nq;
  c.lw = c.Hv < 256 ? c.Hv : 256;
  c.n_vg = c.Hv / c.lw;
  c.n_rows = n_rows; c.n_seqs = n_seqs;
  {
    const int64_t bound = static_cast<int64_t>(n_rows) / c.nq + n_seqs;
    c.nv_max = static_cast<int>(bound < n_rows ? bound : n_rows);
    if (c.nv_max < 1) c.nv_max = 1;
  }
  c.n_groups = c.Hkv / c.kvt;
  c.t_pad = (max_seq_len + 15) / 16 * 16;
  c.MB = d->max_blocks_per_seq; c.NB = d->num_blocks;
  const int sms = device_sm_count();
  // K pass: one CTA per SM, two query-tile slots, up to 8 stages, accumulators of kcols columns
  c.kb = (c.r + 63) / 64;
  c.ksteps = (c.r + 15) / 16;
  c.a_bytes = static_cast<uint32_t>(c.kb) * 16384u;
  c.b_bytes = static_cast<uint32_t>(c.kb) * 2u * c.kcols * 128u;
  c.nbs = 2;
  c.nacc = 512 / c.kcols;
  c.k_tmem = 512;
  {
    const size_t fixed = 1024 + c.nbs * static_cast<size_t>(c.b_bytes) + (4 + 2 * kKTCMaxAcc + 1) * 8;
    int stages = static_cast<int>((200u * 1024u - fixed) / (c.a_bytes + 16u));
    if (stages > 8) stages = 8;
    if (stages < 2) return STARKV_ERR_UNSUPPORTED;
    c.k_stages = stages;
    c.k_smem = fixed + static_cast<size_t>(stages) * (c.a_bytes + 16u);
  }
  c.k_ctas = sms;
  // V pass: lw virtual heads per CTA and mt 128-row M tiles of R (TMEM: mt * lw
  // columns <= 512).  Per token, the V codes are read once per group of
  // virtual heads (Hv / lw groups) and the fp16 weights once per R range (R /
  // (128 mt) ranges): the split with the fewest bytes per token wins (the
  // larger lw on a tie).  The logits, and the weights written over them, are
  // laid out in rows of lw virtual heads.
  {
    const int rpad = (c.R + 127) / 128 * 128;
    int64_t best = -1;
    for (int lw = c.Hv < STARKV_CV_LW_MAX ? c.Hv : STARKV_CV_LW_MAX; lw >= 32 && lw >= c.vpk; lw /= 2)
      for (int mt = 512 / lw; mt >= 1; mt /= 2) {
        if (mt * 128 > rpad && mt > 1) continue;
        const int n_vg = c.Hv / lw;
        const int n_rr = (c.R + mt * 128 - 1) / (mt * 128);
        const int64_t cost = static_cast<int64_t>(n_vg) * c.R * 2 + static_cast<int64_t>(n_rr) * c.Hv * 2;
        if (best >= 0 && cost >= best) continue;
        best = cost;
        c.lw = lw; c.n_vg = n_vg; c.n_rr = n_rr; c.r_range = mt * 128 < rpad ? mt * 128 : rpad;
      }
    c.r_range_pad = c.r_range;
    c.n_chunks = c.r_range_pad / 64;
    c.n_mtiles = c.r_range_pad / 128;
    c.vtile = static_cast<uint32_t>(c.r_range_pad) * 16 * 2;
    c.ltile = 0;   // the weights arrive as fp16 tiles (chunk_weights_kernel)
    c.ptile = static_cast<uint32_t>(c.lw) * 16 * 2;
    c.v_tmem = static_cast<uint32_t>(pow2_ceil(c.n_mtiles * c.lw < 32 ? 32 : c.n_mtiles * c.lw));
    const int per_sm = 512 / static_cast<int>(c.v_tmem) < 2 ? 512 / static_cast<int>(c.v_tmem) : 2;
    // pages per ring stage: at most STARKV_CV_PPS, fewer while a ring of 3 stages would not fit
    c.v_pps = STARKV_CV_PPS < kMaxPPS ? STARKV_CV_PPS : kMaxPPS;
    while (c.v_pps > 1 && 3u * c.v_pps * (c.vtile + c.ltile + c.ptile) > 200u * 1024u / per_sm) --c.v_pps;
    const uint32_t stage = c.v_pps * (c.vtile + c.ltile + c.ptile);
    c.v_stages = static_cast<int>((200u * 1024u / per_sm) / stage);
    if (c.v_stages > STARKV_CV_STAGE_CAP) c.v_stages = STARKV_CV_STAGE_CAP;
    if (c.v_stages < 2) return STARKV_ERR_UNSUPPORTED;
    c.v_smem = 1024 + static_cast<size_t>(c.v_stages) * stage + c.v_stages * sizeof(StageMeta) +
               (3 * c.v_stages + 4) * sizeof(uint64_t) + (c.lw + 128) * sizeof(float);
    c.v_ctas = sms * per_sm / (c.n_rr * c.n_vg);
    if (c.v_ctas < 1) c.v_ctas = 1;
  }
  c.k_slots = c.k_ctas + c.nv_max;
  c.v_slots = c.v_ctas + c.nv_max;
  // finish: tiles of virtual sequences (nq rows each)
  c.up_mt = (c.d + 127) / 128;
  // tiles of up to 256 / nq virtual sequences (64 when shared memory is
  // short); a stage stages at most the partial rows that fit (107 KiB stages),
  // wider tiles read theirs from global memory
  c.up_bt_rows = 256 / c.nq;
  if (c.up_bt_rows > c.nv_max) c.up_bt_rows = c.nv_max;
  for (int tries = 0; tries < 16; ++tries) {
    const int rows = c.up_bt_rows * c.nq;
    c.up_npad = rows < 16 ? 16 : (rows + 15) / 16 * 16;
    const int need = (c.up_bt_rows + c.v_ctas - 1) * c.nq;
    const int cap = static_cast<int>((107u * 1024u - 2u * kFinKC * 128u - 2u * c.up_npad * 128u) / 256u) /
                    kFinZBox * kFinZBox;
    c.up_zrows = (need + kFinZBox - 1) / kFinZBox * kFinZBox;
    if (c.up_zrows > cap) c.up_zrows = cap;
    if (c.up_zrows >= 2 * kFinZBox || c.up_bt_rows == 1) break;
    c.up_bt_rows /= 2;
  }
  if (c.up_zrows < kFinZBox) return STARKV_ERR_UNSUPPORTED;
  c.up_stage_bytes = static_cast<uint32_t>(
      align_up(2u * kFinKC * 128u + 2u * static_cast<size_t>(c.up_npad) * 128u + c.up_zrows * 256u, 1024));
  c.up_smem = 1024 + 2 * static_cast<size_t>(c.up_stage_bytes) + 7 * sizeof(uint64_t) + 3 * kFinMaxRows * 4;
  if (c.up_smem > 220u * 1024u) return STARKV_ERR_UNSUPPORTED;
  c.up_bt = (c.nv_max + c.up_bt_rows - 1) / c.up_bt_rows;
  c.up_ks = 1;
  while (c.up_ks < 8 && c.H * c.up_mt * c.up_bt * c.up_ks * 2 <= sms && c.R / kFinKC >= c.up_ks * 2) c.up_ks *= 2;
  c.up_kpc = ((c.R + c.up_ks * kFinKC - 1) / (c.up_ks * kFinKC)) * kFinKC;
  c.up_tmem = static_cast<uint32_t>(pow2_ceil(c.up_npad < 32 ? 32 : c.up_npad));
  // workspace
  size_t off = 0;
  const size_t nv = static_cast<size_t>(c.nv_max);
  c.status_off = off; off += 256;
  c.prefix_off = off; off = align_up(off + (nv + 1) * 4, 256);
  c.teff_off = off; off = align_up(off + nv * 4, 256);
  c.vs_seq_off = off; off = align_up(off + nv * 4, 256);
  c.vs_row0_off = off; off = align_up(off + nv * 4, 256);
  c.vs_nrows_off = off; off = align_up(off + nv * 4, 256);
  c.vs_len_off = off; off = align_up(off + nv * 4, 256);
  c.qth_off = off; off = align_up(off + nv * 2 * c.Hv * c.r * 2, 256);
  c.logits_off = off; off = align_up(off + nv * c.n_vg * c.t_pad * static_cast<size_t>(c.lw) * 4, 256);
  c.wts_off = off; off = align_up(off + nv * c.n_vg * c.t_pad * static_cast<size_t>(c.lw) * 2, 256);
  c.mpart_off = off; off = align_up(off + static_cast<size_t>(c.k_slots) * c.Hv * 4, 256);
  c.lpart_off = off; off = align_up(off + static_cast<size_t>(c.v_slots) * c.Hv * 4, 256);
  c.n_pc = static_cast<int>((c.t_pad / kBlock + kCwPages - 1) / kCwPages);
  c.lwpart_off = off; off = align_up(off + nv * c.n_pc * c.Hv * 4, 256);
  c.zpart_off = off;
  off = align_up(off + static_cast<size_t>(c.n_rr) * c.H * c.v_slots * c.nq * c.r_range * 4, 256);
  c.total = off;
  return STARKV_OK;
}

starkv_status chunk_prefill(const ChunkPlan& c, const void* q, const void* B_K, const void* B_V, const void* k_cache,
                            const void* v_cache, const int32_t* block_tables, const int32_t* starts,
                            const int32_t* row_offsets, float scale, uint8_t* ws, void* out, cudaStream_t s) {
  int32_t* status = reinterpret_cast<int32_t*>(ws + c.status_off);
  int32_t* prefix = reinterpret_cast<int32_t*>(ws + c.prefix_off);
  int32_t* teff = reinterpret_cast<int32_t*>(ws + c.teff_off);
  int32_t* vs_seq = reinterpret_cast<int32_t*>(ws + c.vs_seq_off);
  int32_t* vs_row0 = reinterpret_cast<int32_t*>(ws + c.vs_row0_off);
  int32_t* vs_nrows = reinterpret_cast<int32_t*>(ws + c.vs_nrows_off);
  int32_t* vs_len = reinterpret_cast<int32_t*>(ws + c.vs_len_off);
  __half* qth = reinterpret_cast<__half*>(ws + c.qth_off);
  float* logits = reinterpret_cast<float*>(ws + c.logits_off);
  float* mpart = reinterpret_cast<float*>(ws + c.mpart_off);
  float* lpart = reinterpret_cast<float*>(ws + c.lpart_off);
  float* lwpart = reinterpret_cast<float*>(ws + c.lwpart_off);
  __half* wts = reinterpret_cast<__half*>(ws + c.wts_off);
  float* zpart = reinterpret_cast<float*>(ws + c.zpart_off);

  CUtensorMap kmap, qmap, vmap, bvmap, zmap;
  if (!encode_kpool_map(&kmap, k_cache, c.r, c.Hkv, c.NB, static_cast<uint32_t>(c.kvt), 16) ||
      !encode_2d_map(&qmap, qth, static_cast<uint64_t>(c.r), static_cast<uint64_t>(c.nv_max) * 2 * c.Hv, 64,
                     static_cast<uint32_t>(c.kcols)) ||
      !encode_vpool_map(&vmap, v_cache, c.R, c.NB, static_cast<uint32_t>(c.n_chunks)) ||
      !encode_2d_map(&bvmap, B_V, static_cast<uint64_t>(c.Hkv) * c.d, static_cast<uint64_t>(c.R), 64, kFinKC) ||
      !encode_f32_rows_map(&zmap, zpart, static_cast<uint64_t>(c.r_range),
                           static_cast<uint64_t>(c.n_rr) * c.H * c.v_slots * c.nq, 64, kFinZBox))
    return STARKV_ERR_CUDA;

  ChunkTableParams tp{starts, row_offsets, vs_seq, vs_row0, vs_nrows, vs_len, c.n_seqs, c.nv_max, c.log2nq};
  if (launch(chunk_table_kernel, dim3(1), dim3(256), 0, s, 1, tp) != cudaSuccess) return STARKV_ERR_CUDA;

  AbsorbParams ap{};
  std::memset(&ap, 0, sizeof(ap));
  ap.q = static_cast<const __half*>(q);
  ap.B_K = static_cast<const __half*>(B_K);
  ap.seq_lens = vs_len;
  ap.qt = nullptr; ap.qth = qth; ap.prefix = prefix; ap.teff = teff; ap.status = status;
  ap.mpart_init = mpart;
  ap.n_mpart = c.k_slots * c.Hv;
  ap.B = c.nv_max; ap.H = c.H; ap.d = c.d; ap.r = c.r; ap.cap = c.t_pad;
  {
    int lg = 0;
    while ((c.Hkv << lg) < c.H) ++lg;
    ap.log2G = lg;
  }
  ap.coef = scale * kLog2e;
  ap.vs_row0 = vs_row0; ap.vs_nrows = vs_nrows; ap.log2nq = c.log2nq;
  if (launch_prep(c.d, nullptr, &ap, c.nv_max << c.log2nq, s) != STARKV_OK) return STARKV_ERR_CUDA;

  KPassChunkParams kp{};
  kp.tables = block_tables; kp.vs_seq = vs_seq; kp.vs_nrows = vs_nrows; kp.teff = teff; kp.prefix = prefix;
  kp.logits = logits; kp.mpart = mpart; kp.status = status;
  kp.B = c.nv_max; kp.MB = c.MB; kp.NB = c.NB; kp.t_pad = c.t_pad;
  kp.Hv = c.Hv; kp.n_vg = c.n_vg; kp.n_groups = c.n_groups; kp.log2nq = c.log2nq;
  kp.log2lw = 0;
  while ((1 << kp.log2lw) < c.lw) ++kp.log2lw;
  kp.ksteps = c.ksteps; kp.kb = c.kb; kp.nacc = c.nacc; kp.nbs = c.nbs; kp.stages = c.k_stages;
  kp.a_bytes = c.a_bytes; kp.b_bytes = c.b_bytes; kp.tmem_cols = c.k_tmem;
  kp.drop_stage = g_drop_k_stage.load(std::memory_order_relaxed);
  if (launch_kpass_chunk(c.vpk, c.k_smem, c.k_ctas, kmap, qmap, kp, s) != cudaSuccess) return STARKV_ERR_CUDA;

  ChunkWeightsParams wp{logits, wts,  mpart,   teff,  prefix,   lwpart,
                        c.nv_max, c.Hv, c.n_vg, c.lw, kp.log2lw, c.t_pad, c.k_ctas, c.n_pc};
  if (launch(chunk_weights_kernel, dim3(c.nv_max, c.n_pc, c.n_vg), dim3(256), 0, s, 1, wp) != cudaSuccess)
    return STARKV_ERR_CUDA;

  VPassParams vp{};
  std::memset(&vp, 0, sizeof(vp));
  vp.tables = block_tables; vp.row_seq = vs_seq; vp.teff = teff; vp.prefix = prefix; vp.logits = logits;
  vp.mpart = mpart; vp.zpart = zpart; vp.lpart = lpart; vp.status = status;
  vp.B = c.nv_max; vp.H = c.H; vp.npad = c.lw; vp.MB = c.MB; vp.NB = c.NB; vp.R = c.R;
  vp.t_pad = c.t_pad; vp.r_range = c.r_range; vp.n_rr = c.n_rr; vp.v_slots = c.v_slots;
  vp.stages = c.v_stages; vp.n_chunks = c.n_chunks; vp.n_mtiles = c.n_mtiles; vp.tmem_cols = c.v_tmem;
  vp.vtile_bytes = c.vtile; vp.ltile_bytes = c.ltile; vp.ptile_bytes = c.ptile; vp.pps = c.v_pps; vp.wts = wts;
  vp.Hv = c.Hv; vp.n_vg = c.n_vg; vp.log2nq = c.log2nq; vp.lw = c.lw;
  if (!set_smem(vpass_kernel<true>, c.v_smem)) return STARKV_ERR_CUDA;
  if (launch(vpass_kernel<true>, dim3(c.v_ctas, c.n_rr * c.n_vg), dim3(kVThreads), c.v_smem, s, 1, vmap, vp) !=
      cudaSuccess)
    return STARKV_ERR_CUDA;

  FinishParams fp{};
  std::memset(&fp, 0, sizeof(fp));
  fp.out = static_cast<__half*>(out);
  fp.zpart = zpart; fp.lpart = lpart; fp.prefix = prefix;
  fp.B = c.nv_max; fp.H = c.H; fp.d = c.d; fp.R = c.R;
  fp.log2G = ap.log2G;
  fp.r_range = c.r_range; fp.v_slots = c.v_slots; fp.v_grid = c.v_ctas;
  fp.n_mt = c.up_mt; fp.bt_rows = c.up_bt_rows; fp.k_per_cta = c.up_kpc; fp.npad = c.up_npad;
  fp.stages = 2; fp.zrows = c.up_zrows; fp.stage_bytes = c.up_stage_bytes; fp.tmem_cols = c.up_tmem;
  fp.vs_row0 = vs_row0; fp.vs_nrows = vs_nrows; fp.log2nq = c.log2nq; fp.Hv = c.Hv; fp.lwpart = lwpart; fp.n_pc = c.n_pc;
  if (!set_smem(finish_kernel, c.up_smem)) return STARKV_ERR_CUDA;
  if (launch(finish_kernel, dim3(c.H * c.up_mt * c.up_bt, c.up_ks), dim3(kFinThreads), c.up_smem, s, c.up_ks,
             bvmap, zmap, fp) != cudaSuccess)
    return STARKV_ERR_CUDA;
  return STARKV_OK;
}
}  // namespace

size_t starkv_prefill_workspace_bytes(const starkv_layer_desc* desc, int32_t n_seqs, int32_t n_rows,
                                      int32_t max_seq_len) {
  DecodePlan pl{};
  if (n_seqs < 0 || n_rows < 0 || make_plan(desc, n_rows, max_seq_len, &pl) != STARKV_OK) return 0;
  ChunkPlan cp{};
  if (chunk_eligible(desc)) return make_chunk_plan(desc, n_seqs, n_rows, max_seq_len, &cp) == STARKV_OK ? cp.total : 0;
  return prefill_rows_offset(pl) + align_up(static_cast<size_t>(n_rows) * 8, 256);
}

starkv_status starkv_paged_prefill(const starkv_layer_desc* desc, int32_t n_seqs, int32_t n_rows, int32_t max_seq_len,
                                   const void* q, const void* B_K, const void* B_V, const void* k_cache,
                                   const void* v_cache, const int32_t* block_tables, const int32_t* starts,
                                   const int32_t* row_offsets, float scale, void* workspace, size_t workspace_bytes,
                                   void* out, void* stream) {
  DecodePlan pl{};
  if (n_seqs < 0 || n_rows < 0) return STARKV_ERR_INVALID_ARG;
  starkv_status st = make_plan(desc, n_rows, max_seq_len, &pl);
  if (st != STARKV_OK) return st;
  if (n_rows == 0) return clear_status(workspace, workspace_bytes, stream);
  if (n_seqs == 0 || !starts || !row_offsets || (reinterpret_cast<uintptr_t>(starts) & 3u) ||
      (reinterpret_cast<uintptr_t>(row_offsets) & 3u))
    return STARKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ChunkPlan cp{};
  if (chunk_eligible(desc)) {
    if (make_chunk_plan(desc, n_seqs, n_rows, max_seq_len, &cp) != STARKV_OK) return STARKV_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < cp.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
      return STARKV_ERR_WORKSPACE;
    if (!q || !B_K || !B_V || !k_cache || !v_cache || !block_tables || !out || !aligned16(q) || !aligned16(B_K) ||
        !aligned16(B_V) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) || !(std::isfinite(scale) && scale > 0.f))
      return STARKV_ERR_INVALID_ARG;
    return chunk_prefill(cp, q, B_K, B_V, k_cache, v_cache, block_tables, starts, row_offsets, scale,
                         static_cast<uint8_t*>(workspace), out, s);
  }
  const size_t need = prefill_rows_offset(pl) + align_up(static_cast<size_t>(n_rows) * 8, 256);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return STARKV_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* row_seq = reinterpret_cast<int32_t*>(ws + prefill_rows_offset(pl));
  int32_t* row_len = row_seq + n_rows;
  PrefillRowsParams rp{starts, row_offsets, row_seq, row_len, n_seqs, n_rows};
  if (launch(prefill_rows_kernel, dim3((n_rows + 255) / 256), dim3(256), 0, s, 1, rp) != cudaSuccess)
    return STARKV_ERR_CUDA;
  return decode_impl(desc, n_rows, max_seq_len, q, B_K, B_V, k_cache, v_cache, block_tables, row_len, scale,
                     workspace, workspace_bytes, out, stream, nullptr, row_seq);
}

starkv_status starkv_paged_decode_profiled(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len,
                                           const void* q, const void* B_K, const void* B_V, const void* k_cache,
                                           const void* v_cache, const int32_t* block_tables,
                                           const int32_t* seq_lens, float scale, void* workspace,
                                           size_t workspace_bytes, void* out, void* stream,
                                           void* const* stage_events) {
  return decode_impl(desc, batch, max_seq_len, q, B_K, B_V, k_cache, v_cache, block_tables, seq_lens, scale,
                     workspace, workspace_bytes, out, stream, stage_events);
}

// ---------------------------------------------------------------------------
// Decode without a caller-provided workspace.  Some callers cannot allocate
// device memory when they decode: a serving engine that reserved nearly all of
// the GPU's memory for its paged KV pool up front (a later cudaMalloc fails or
// eats into the pool), or a plain C host that has no allocator of its own to
// hand out scratch.  For them the scratch lives in this fixed device array,
// which every GPU that loads the library holds until the process exits.
#define STARKV_STATIC_WS_BYTES (64ull << 20)
static __device__ __align__(256) uint8_t g_starkv_static_ws[STARKV_STATIC_WS_BYTES];

namespace {
std::mutex g_static_ws_mu;
void* g_static_ws_ptr[64] = {};

// Device address of the array on the current device, looked up once per device
// (host code may not use the symbol itself: it names a host-side stand-in).
void* static_ws_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_static_ws_mu);
  if (!g_static_ws_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_starkv_static_ws) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return nullptr;
    }
    g_static_ws_ptr[dev] = ptr;
  }
  return g_static_ws_ptr[dev];
}
}  // namespace

starkv_status starkv_paged_decode_static(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len,
                                         const void* q, const void* B_K, const void* B_V, const void* k_cache,
                                         const void* v_cache, const int32_t* block_tables,
                                         const int32_t* seq_lens, float scale, void* out, void* stream) {
  DecodePlan pl{};
  starkv_status st = make_plan(desc, batch, max_seq_len, &pl);
  if (st != STARKV_OK) return st;
  if (pl.ws.total_bytes > STARKV_STATIC_WS_BYTES) return STARKV_ERR_WORKSPACE;
  if (batch == 0) return decode_impl(desc, batch, max_seq_len, q, B_K, B_V, k_cache, v_cache, block_tables,
                                     seq_lens, scale, nullptr, 0, out, stream, nullptr);
  void* ws = static_ws_address();
  if (!ws) return STARKV_ERR_CUDA;
  return decode_impl(desc, batch, max_seq_len, q, B_K, B_V, k_cache, v_cache, block_tables, seq_lens, scale, ws,
                     STARKV_STATIC_WS_BYTES, out, stream, nullptr);
}

starkv_status starkv_decode_check(const void* workspace, void* stream, int32_t* flags_out) {
  if (!workspace || !flags_out) return STARKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t flags = 0;
  if (cudaMemcpyAsync(&flags, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return STARKV_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return STARKV_ERR_CUDA;
  *flags_out = flags;
  if (flags & STARKV_FLAG_TIMEOUT) return STARKV_ERR_TIMEOUT;
  if (flags) return STARKV_ERR_DEVICE_CHECK;
  return STARKV_OK;
}

}  // extern "C"
