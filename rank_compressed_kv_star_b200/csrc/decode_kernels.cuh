// Decode kernels of the STAR-KV paged low-rank cache (sm_100a).
//
// One decode is five launches on the caller's stream:
//   1. absorb      q~ = log2(e)*scale * q . B_K[h]^T; page prefix sums; status reset
//   2. kpass       base-2 logits s = q~ . c_K over the K pages, per-segment max
//   3. reduce      per (b, h): global max M of the logits
//   4. vpass       Z = sum_t w c_V on tcgen05 tensor cores with w = fp16(exp2(s - M)),
//                  and the normaliser L = sum_t w
//   5. upproj      out_h = (Z_h . B_V[:, h*d:(h+1)*d]) / L -> fp16
//
// The formulation (head-wise K with the query absorbed, joint V applied after
// the weighted sum of codes) follows the STAR-KV description in the Proxima
// README ("Low-rank KV Cache Compression for vLLM", method paragraph): K is
// decomposed per head, V jointly across heads, and both are stored as codes in
// a paged format of 16-token blocks.
//
// Work partition of the two streaming passes.  All pages of all sequences are
// laid end to end (sequence b owns pages [prefix[b], prefix[b+1])) and CTA i of
// a G-CTA grid takes pages [floor(i*P/G), floor((i+1)*P/G)), with G <= P so no
// range is empty.  A CTA's range can cross sequence boundaries; it emits one
// partial result per (sequence, CTA) pair into slot b + i, which is unique
// because ranges are contiguous and ordered.  The split reduction and the
// up-projection visit the CTAs overlapping sequence b in increasing i, so every
// result is independent of which physical pages hold the codes.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "../../include/starkv.h"

namespace starkv {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kBlock = 16;  // tokens per page

struct Partition {
  int64_t P;   // total pages
  int32_t G;   // CTAs that hold work, min(grid, P)
};

__device__ __forceinline__ int64_t part_begin(int64_t i, const Partition& pt) {
  return (i * pt.P) / pt.G;
}
// Largest CTA index whose range starts at or before page x (0 <= x < P).
__device__ __forceinline__ int32_t part_owner(int64_t x, const Partition& pt) {
  int64_t i = ((x + 1) * pt.G + pt.P - 1) / pt.P - 1;
  return static_cast<int32_t>(i < pt.G - 1 ? i : pt.G - 1);
}
// Largest b with prefix[b] <= x (prefix is non-decreasing, prefix[0] = 0).
__device__ __forceinline__ int32_t seq_of_page(const int32_t* prefix, int32_t B, int64_t x) {
  int32_t lo = 0, hi = B - 1;
  while (lo < hi) {
    int32_t mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void set_flag(int32_t* status, int32_t f) { atomicOr(status, f); }

// Timeout at pipeline wait `site`: the timeout bit plus a per-site bit (8..15)
// that tells where the pipeline stopped.
enum WaitSite : int32_t {
  kSiteKEmpty = 0, kSiteKFull = 1, kSiteVEmpty = 2, kSiteVPready = 3, kSiteVTfree = 4,
  kSiteVFull = 5, kSiteVZdone = 6, kSiteVMdone = 7
};
__device__ __forceinline__ void set_timeout(int32_t* status, WaitSite site) {
  atomicOr(status, STARKV_FLAG_TIMEOUT | (1 << (8 + site)));
}

// ====================================================================== absorb
struct AbsorbParams {
  const __half* q;        // [B][H][d]
  const __half* B_K;      // [H][r][d]
  const int32_t* seq_lens;
  float* qt;              // [B][H][r]
  int32_t* prefix;        // [B+1]
  int32_t* teff;          // [B] clamped lengths
  int32_t* status;
  int B, H, d, r, cap;    // cap = min(max_seq_len, max_blocks_per_seq*16)
  float coef;             // scale * log2(e)
};

// grid (H), 256 threads.  CTA 0 also writes the page prefix sums and resets the
// status word (every later kernel of the decode runs after this one).
__global__ void __launch_bounds__(256) absorb_kernel(AbsorbParams p) {
  const int h = blockIdx.x;
  const int tid = threadIdx.x;
  if (h == 0) {
    __shared__ int32_t part[256];
    __shared__ int32_t bad;
    if (tid == 0) bad = 0;
    __syncthreads();
    const int per = (p.B + 255) / 256;
    const int b0 = tid * per;
    int32_t s = 0;
    for (int b = b0; b < b0 + per && b < p.B; ++b) {
      int32_t T = p.seq_lens[b];
      if (T < 0 || T > p.cap) { bad = 1; T = T < 0 ? 0 : p.cap; }
      p.teff[b] = T;
      s += (T + kBlock - 1) / kBlock;
    }
    part[tid] = s;
    __syncthreads();
    if (tid == 0) {
      int32_t acc = 0;
      for (int i = 0; i < 256; ++i) { int32_t v = part[i]; part[i] = acc; acc += v; }
      p.prefix[p.B] = acc;
      *p.status = bad ? STARKV_FLAG_BAD_SEQ_LEN : 0;
    }
    __syncthreads();
    int32_t acc = part[tid];
    for (int b = b0; b < b0 + per && b < p.B; ++b) {
      p.prefix[b] = acc;
      acc += (p.teff[b] + kBlock - 1) / kBlock;
    }
  }
  // q~[b,h,i] = coef * sum_j q[b,h,j] * B_K[h][i][j]
  const int i = tid % p.r;
  const int bpar = 256 / p.r;
  const int bs = tid / p.r;
  if (bs >= bpar) return;
  const __half* brow = p.B_K + (static_cast<size_t>(h) * p.r + i) * p.d;
  for (int b = bs; b < p.B; b += bpar) {
    const __half* qrow = p.q + (static_cast<size_t>(b) * p.H + h) * p.d;
    float acc = 0.f;
    for (int j = 0; j < p.d; j += 8) {
      const uint4 bw = *reinterpret_cast<const uint4*>(brow + j);
      const uint4 qw = *reinterpret_cast<const uint4*>(qrow + j);
      const __half2* b2 = reinterpret_cast<const __half2*>(&bw);
      const __half2* q2 = reinterpret_cast<const __half2*>(&qw);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 bf = __half22float2(b2[u]);
        const float2 qf = __half22float2(q2[u]);
        acc = fmaf(qf.x, bf.x, acc);
        acc = fmaf(qf.y, bf.y, acc);
      }
    }
    p.qt[(static_cast<size_t>(b) * p.H + h) * p.r + i] = acc * p.coef;
  }
}

// ======================================================================= kpass
struct KPassParams {
  const __half* k_cache;      // [NB][16][H][r]
  const int32_t* tables;      // [B][MB]
  const int32_t* teff;        // [B]
  const int32_t* prefix;      // [B+1]
  const float* qt;            // [B][H][r]
  float* logits;              // [B][t_pad][H]
  float* mpart;               // [k_slots][H]: max of the base-2 logits per segment
  int32_t* status;
  int B, H, log2H, r, MB, NB, t_pad;
  int tps;                    // tokens per ring stage
  int stages;
  uint32_t stage_bytes;       // tps*H*r*2
};

constexpr int kKConsumers = 256;            // 8 warps of dot products
constexpr int kKThreads = kKConsumers + 32; // + one producer warp

struct StageMeta { int32_t b, t0, nt, flags; };

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)),
        "l"(*reinterpret_cast<uint64_t*>(&c)));
  return *reinterpret_cast<float2*>(&d);
}

// First chunk a thread visits, chosen so that the 8 threads sharing a
// shared-memory wavefront (8 consecutive rows of r*2 bytes, 16-byte reads)
// hit 8 different bank groups: bank group of (row, chunk) is
// (row*CP + chunk) mod 8 with CP = r/8 chunks per row.
__device__ __forceinline__ int chunk_rotation(int tid, int cp, int L) {
  if (L > 1 || cp % 8 == 0) return tid & 7;
  if (cp % 4 == 0) return (tid >> 1) & 3;
  return (tid >> 2) & 1;
}

// One (token, head) dot product of length r per L threads: each thread reads
// CPT 16-byte chunks (8 codes) of its row in a rotated order and accumulates
// with packed fp32 FMAs against its head's absorbed query held in registers.
// The head of a thread is fixed because (kKConsumers / L) is a multiple of H.
template <int L, int CPT>
__global__ void __launch_bounds__(kKThreads, 1) kpass_kernel(KPassParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int S = p.stages;
  uint8_t* ring = smem;
  StageMeta* meta = reinterpret_cast<StageMeta*>(smem + static_cast<size_t>(S) * p.stage_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(meta + S);
  uint64_t* empty = full + S;
  float* red = reinterpret_cast<float*>(empty + S);         // [kKConsumers / L]
  __shared__ volatile int32_t abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kKConsumers / 32); }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  Partition pt;
  pt.P = p.prefix[p.B];
  pt.G = static_cast<int32_t>(pt.P < gridDim.x ? pt.P : gridDim.x);
  const int cta = blockIdx.x;
  const bool has_work = cta < pt.G;

  if (warp == kKConsumers / 32) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    const uint32_t tok_bytes = static_cast<uint32_t>(p.H) * p.r * 2;
    uint32_t k = 0;
    bool ok = true;
    if (has_work) {
      const int64_t p0 = part_begin(cta, pt), p1 = part_begin(cta + 1, pt);
      int32_t b = seq_of_page(p.prefix, p.B, p0);
      for (int64_t pg_g = p0; pg_g < p1 && ok; ++pg_g) {
        while (p.prefix[b + 1] <= pg_g) ++b;
        const int32_t pg = static_cast<int32_t>(pg_g - p.prefix[b]);
        const int32_t T = p.teff[b];
        int32_t phys = p.tables[static_cast<size_t>(b) * p.MB + pg];
        if (phys < 0 || phys >= p.NB) { set_flag(p.status, STARKV_FLAG_BAD_BLOCK_ID); phys = 0; }
        const int32_t tend = min(pg * kBlock + kBlock, T);
        for (int32_t t0 = pg * kBlock; t0 < tend; t0 += p.tps, ++k) {
          const int s = k % S;
          if (k >= static_cast<uint32_t>(S) && !mbar_wait(&empty[s], ((k / S) - 1) & 1)) { ok = false; break; }
          const int32_t nt = min(p.tps, tend - t0);
          meta[s] = StageMeta{b, t0, nt, 0};
          const uint32_t bytes = static_cast<uint32_t>(nt) * tok_bytes;
          mbar_arrive_expect_tx(&full[s], bytes);
          const __half* src = p.k_cache + (static_cast<size_t>(phys) * kBlock + (t0 - pg * kBlock)) *
                                              static_cast<size_t>(p.H) * p.r;
          bulk_g2s(ring + static_cast<size_t>(s) * p.stage_bytes, src, bytes, &full[s], pol);
        }
      }
    }
    if (ok) {
      const int s = k % S;
      if (k >= static_cast<uint32_t>(S) && !mbar_wait(&empty[s], ((k / S) - 1) & 1)) ok = false;
      if (ok) { meta[s] = StageMeta{-1, 0, 0, 0}; mbar_arrive(&full[s]); }
    }
    if (!ok) {
      set_timeout(p.status, kSiteKEmpty);
      abort_flag = 1;
      // let copies already in flight land before the CTA can exit
      const uint32_t first = k > static_cast<uint32_t>(S) ? k - S : 0;
      for (uint32_t kk = first; kk < k; ++kk) mbar_wait(&full[kk % S], (kk / S) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  constexpr int kPairsPerPass = kKConsumers / L;
  const int pair0 = tid / L;
  const int sub = tid % L;
  const int head = pair0 & (p.H - 1);
  const int cp = p.r >> 3;                  // 16-byte chunks per (token, head) row
  const int rot = chunk_rotation(tid, cp, L);
  const int passes = (p.tps * p.H + kPairsPerPass - 1) / kPairsPerPass;
  float2 qv[CPT * 4];
  float m = -INFINITY;
  int cur_b = -1;

  for (uint32_t k = 0;; ++k) {
    const int s = k % S;
    if (!mbar_wait(&full[s], (k / S) & 1) || abort_flag) {
      set_timeout(p.status, kSiteKFull);
      break;
    }
    const StageMeta mt = meta[s];
    if (mt.b != cur_b || mt.b < 0) {   // new sequence, or the end marker (b < 0)
      if (cur_b >= 0) {
        // per-segment max for every head: slot = sequence + CTA
        if (sub == 0) red[pair0] = m;
        named_bar_sync(1, kKConsumers);
        if (tid < p.H) {
          float M = -INFINITY;
          for (int g = tid; g < kPairsPerPass; g += p.H) M = fmaxf(M, red[g]);
          p.mpart[static_cast<size_t>(cur_b + cta) * p.H + tid] = M;
        }
        named_bar_sync(1, kKConsumers);
      }
      if (mt.b < 0) break;
      cur_b = mt.b;
      m = -INFINITY;
      const float* qsrc = p.qt + (static_cast<size_t>(cur_b) * p.H + head) * p.r;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const int cc = c + rot < CPT ? c + rot : c + rot - CPT;
        const int ch = sub * CPT + cc;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          qv[c * 4 + u] = ch < cp ? make_float2(qsrc[ch * 8 + 2 * u], qsrc[ch * 8 + 2 * u + 1])
                                  : make_float2(0.f, 0.f);
      }
    }
    const uint8_t* st = ring + static_cast<size_t>(s) * p.stage_bytes;
    for (int ps = 0; ps < passes; ++ps) {
      const int pair = ps * kPairsPerPass + pair0;
      const int t = pair >> p.log2H;     // token within the stage; pair & (H-1) == head
      const bool valid = t < mt.nt;
      float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
      if (valid) {
        const uint8_t* row = st + static_cast<size_t>(pair) * p.r * 2;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          const int cc = c + rot < CPT ? c + rot : c + rot - CPT;
          const int ch = sub * CPT + cc;
          if (ch < cp) {
            const uint4 w = *reinterpret_cast<const uint4*>(row + ch * 16);
            const __half2* h2 = reinterpret_cast<const __half2*>(&w);
            a0 = ffma2(__half22float2(h2[0]), qv[c * 4 + 0], a0);
            a1 = ffma2(__half22float2(h2[1]), qv[c * 4 + 1], a1);
            a2 = ffma2(__half22float2(h2[2]), qv[c * 4 + 2], a2);
            a3 = ffma2(__half22float2(h2[3]), qv[c * 4 + 3], a3);
          }
        }
      }
      float acc = ((a0.x + a0.y) + (a1.x + a1.y)) + ((a2.x + a2.y) + (a3.x + a3.y));
#pragma unroll
      for (int o = L / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (valid) {
        if (sub == 0)
          p.logits[(static_cast<size_t>(cur_b) * p.t_pad + mt.t0 + t) * p.H + head] = acc;
        m = fmaxf(m, acc);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

// ====================================================================== reduce
struct ReduceParams {
  const float* mpart;     // [k_slots][H]
  const int32_t* prefix;  // [B+1]
  float* mx;              // [B][H]: max of the base-2 logits of each sequence and head
  int B, H, k_grid;
};

__global__ void __launch_bounds__(256) reduce_kernel(ReduceParams p) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= p.B * p.H) return;
  const int b = idx / p.H, h = idx % p.H;
  const int32_t f0 = p.prefix[b], f1 = p.prefix[b + 1];
  if (f1 == f0) { p.mx[idx] = 0.f; return; }
  Partition pt;
  pt.P = p.prefix[p.B];
  pt.G = static_cast<int32_t>(pt.P < p.k_grid ? pt.P : p.k_grid);
  const int32_t i0 = part_owner(f0, pt), i1 = part_owner(f1 - 1, pt);
  float M = -INFINITY;
  for (int32_t i = i0; i <= i1; ++i) M = fmaxf(M, p.mpart[static_cast<size_t>(b + i) * p.H + h]);
  p.mx[idx] = M;
}

// ======================================================================= vpass
// Z^T (R-range rows x heads) += C_V^T (R-range x 16 tokens) . P^T (16 x heads)
// per page, with A = the V page slice as an MN-major 128B-swizzled operand
// (exactly the layout TMA writes for 64-element x 16-token boxes) and B = the
// fp16 attention weights in a K-major, unswizzled layout written by the
// P warps.  The accumulator lives in tensor memory: one 128-lane x npad-column
// block per 128 rows of the R range.
struct VPassParams {
  const int32_t* tables;
  const int32_t* teff;
  const int32_t* prefix;
  const float* logits;    // [B][t_pad][H]
  const float* mx;        // [B][H]
  float* zpart;           // [n_rr][v_slots][H][r_range]: sum_t w c_V per segment
  float* lpart;           // [v_slots][H]: sum_t w per segment (written by R range 0)
  int32_t* status;
  int B, H, npad, MB, NB, R, t_pad, r_range, n_rr, v_slots, stages;
  int n_chunks;           // 64-wide chunks per R range (r_range_pad/64); the last range may hold fewer
  int n_mtiles;           // r_range_pad / 128
  uint32_t tmem_cols;
  uint32_t vtile_bytes;   // r_range_pad*16*2
  uint32_t ltile_bytes;   // 16*H*4
  uint32_t ptile_bytes;   // npad*16*2
};

constexpr int kVThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 weights + epilogue
constexpr int32_t kFirst = 1, kLast = 2;

__global__ void __launch_bounds__(kVThreads, 1)
vpass_kernel(const __grid_constant__ CUtensorMap vmap, VPassParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  uint8_t* vtiles = smem;                                               // S x vtile_bytes (1024-aligned)
  uint8_t* ltiles = vtiles + static_cast<size_t>(S) * p.vtile_bytes;    // S x ltile_bytes
  uint8_t* ptiles = ltiles + static_cast<size_t>(S) * p.ltile_bytes;    // S x ptile_bytes
  StageMeta* meta = reinterpret_cast<StageMeta*>(ptiles + static_cast<size_t>(S) * p.ptile_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(meta + S);
  uint64_t* pready = full + S;
  uint64_t* empty = pready + S;
  uint64_t* zdone = empty + S;
  uint64_t* tfree = zdone + 1;
  uint64_t* mdone = tfree + 1;
  float* sM = reinterpret_cast<float*>(mdone + 1);                      // [npad]
  float* sRed = sM + p.npad;                                            // [128]
  __shared__ uint32_t taddr_s;
  __shared__ volatile int32_t abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Partition pt;
  pt.P = p.prefix[p.B];
  pt.G = static_cast<int32_t>(pt.P < gridDim.x ? pt.P : gridDim.x);
  const int cta = blockIdx.x;
  const int rr = blockIdx.y;
  if (cta >= pt.G) return;  // uniform across the CTA: nothing allocated yet

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&pready[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(zdone, 1);
    mbar_init(tfree, 128);
    mbar_init(mdone, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&taddr_s, p.tmem_cols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = taddr_s;

  const int64_t p0 = part_begin(cta, pt), p1 = part_begin(cta + 1, pt);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&vmap);
      const uint64_t pol_codes = policy_evict_first();
      const uint64_t pol_logits = policy_evict_first();
      uint32_t k = 0;
      bool ok = true;
      int32_t b = seq_of_page(p.prefix, p.B, p0);
      const int c_base = rr * (p.r_range / 64);
      const int n_ch = min(p.n_chunks, (p.R - rr * p.r_range + 63) / 64);
      for (int64_t pg_g = p0; pg_g < p1; ++pg_g, ++k) {
        while (p.prefix[b + 1] <= pg_g) ++b;
        const int32_t pg = static_cast<int32_t>(pg_g - p.prefix[b]);
        const int32_t npg = p.prefix[b + 1] - p.prefix[b];
        const int32_t T = p.teff[b];
        int32_t phys = p.tables[static_cast<size_t>(b) * p.MB + pg];
        if (phys < 0 || phys >= p.NB) { set_flag(p.status, STARKV_FLAG_BAD_BLOCK_ID); phys = 0; }
        const int s = k % S;
        if (k >= static_cast<uint32_t>(S) && !mbar_wait(&empty[s], ((k / S) - 1) & 1)) { ok = false; break; }
        int32_t fl = 0;
        if (pg_g == p0 || pg == 0) fl |= kFirst;
        if (pg_g == p1 - 1 || pg == npg - 1) fl |= kLast;
        meta[s] = StageMeta{b, pg * kBlock, min(kBlock, T - pg * kBlock), fl};
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(n_ch) * 2048u + p.ltile_bytes);
        uint8_t* vt = vtiles + static_cast<size_t>(s) * p.vtile_bytes;
        for (int c = 0; c < n_ch; ++c)
          tma_load_2d(vt + c * 2048, &vmap, (c_base + c) * 64, phys * kBlock, &full[s], pol_codes);
        bulk_g2s(ltiles + static_cast<size_t>(s) * p.ltile_bytes,
                 p.logits + (static_cast<size_t>(b) * p.t_pad + pg * kBlock) * p.H, p.ltile_bytes,
                 &full[s], pol_logits);
      }
      if (ok) {
        const int s = k % S;
        if (k >= static_cast<uint32_t>(S) && !mbar_wait(&empty[s], ((k / S) - 1) & 1)) ok = false;
        if (ok) { meta[s] = StageMeta{-1, 0, 0, 0}; mbar_arrive(&full[s]); }
      }
      if (!ok) {
        set_timeout(p.status, kSiteVEmpty);
        abort_flag = 1;
        const uint32_t first = k > static_cast<uint32_t>(S) ? k - S : 0;
        for (uint32_t kk = first; kk < k; ++kk) mbar_wait(&full[kk % S], (kk / S) & 1);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, p.npad, /*a_mn_major=*/true, /*b_mn_major=*/false);
      const uint32_t lbo_b = static_cast<uint32_t>(p.npad / 8) * 128u;
      uint32_t seg = 0;
      uint32_t accumulate = 0;
      for (uint32_t k = 0;; ++k) {
        const int s = k % S;
        if (!mbar_wait(&pready[s], (k / S) & 1) || abort_flag) { set_timeout(p.status, kSiteVPready); break; }
        const StageMeta mt = meta[s];
        if (mt.b < 0) break;
        if (mt.flags & kFirst) {
          if (seg > 0 && !mbar_wait(tfree, (seg - 1) & 1)) { set_timeout(p.status, kSiteVTfree); break; }
          accumulate = 0;
        }
        tc_fence_after();
        const uint32_t va = smem_u32(vtiles + static_cast<size_t>(s) * p.vtile_bytes);
        const uint32_t pa = smem_u32(ptiles + static_cast<size_t>(s) * p.ptile_bytes);
        const uint64_t bdesc = smem_desc(pa, lbo_b, 128u, kSwizzleNone);
        for (int m = 0; m < p.n_mtiles; ++m) {
          const uint64_t adesc = smem_desc(va + m * 4096u, 2048u, 1024u, kSwizzle128B);
          umma_f16_ss(taddr + static_cast<uint32_t>(m * p.npad), adesc, bdesc, idesc, accumulate);
        }
        accumulate = 1;
        umma_commit(&empty[s]);
        if (mt.flags & kLast) { umma_commit(zdone); ++seg; }
      }
      // every MMA issued has completed before the CTA can release TMEM
      umma_commit(mdone);
      if (!mbar_wait(mdone, 0)) set_timeout(p.status, kSiteVMdone);
    }
  } else {
    // ------------------------------------------ weights + epilogue (128 thr)
    const int et = tid - 64;             // 0..127
    const int q = warp & 3;              // TMEM lane quarter of this warp
    const uint32_t lbo_b = static_cast<uint32_t>(p.npad / 8) * 128u;
    // this thread's weights: head h_w (fixed), tokens t_w0, t_w0 + t_step, ...
    const int h_w = et % p.npad;
    const int t_w0 = et / p.npad;
    const int t_step = 128 / p.npad;
    float lsum = 0.f;
    uint32_t seg = 0;
    for (uint32_t k = 0;; ++k) {
      const int s = k % S;
      if (!mbar_wait(&full[s], (k / S) & 1) || abort_flag) {
        set_timeout(p.status, kSiteVFull);
        abort_flag = 1;
        break;
      }
      const StageMeta mt = meta[s];
      if (mt.b < 0) { mbar_arrive(&pready[s]); break; }
      if (mt.flags & kFirst) {
        named_bar_sync(2, 128);  // everyone is done with the previous segment's max
        for (int h = et; h < p.npad; h += 128)
          sM[h] = h < p.H ? p.mx[static_cast<size_t>(mt.b) * p.H + h] : 0.f;
        named_bar_sync(2, 128);
        lsum = 0.f;
      }
      const float* lt = reinterpret_cast<const float*>(ltiles + static_cast<size_t>(s) * p.ltile_bytes);
      uint8_t* pt_s = ptiles + static_cast<size_t>(s) * p.ptile_bytes;
      const float m_h = sM[h_w];
      for (int t = t_w0; t < kBlock; t += t_step) {
        // unnormalised weight exp2(s - M) <= 1, rounded to fp16 for the MMA; the
        // normaliser sums exactly the rounded weights
        __half w = __float2half_rn(0.f);
        if (t < mt.nt && h_w < p.H) w = __float2half_rn(exp2f(lt[t * p.H + h_w] - m_h));
        lsum += __half2float(w);
        const uint32_t off = static_cast<uint32_t>(t >> 3) * lbo_b + static_cast<uint32_t>(h_w >> 3) * 128u +
                             static_cast<uint32_t>(h_w & 7) * 16u + static_cast<uint32_t>(t & 7) * 2u;
        *reinterpret_cast<__half*>(pt_s + off) = w;
      }
      if (mt.nt < kBlock) {
        // tokens past the sequence end: zero their rows of the V tile so that
        // whatever the unused slots hold (NaN included) contributes exactly 0
        uint8_t* vt = vtiles + static_cast<size_t>(s) * p.vtile_bytes;
        const int nrows = kBlock - mt.nt;
        const int n_ch = min(p.n_chunks, (p.R - rr * p.r_range + 63) / 64);
        const int nst = n_ch * nrows * 8;  // 16-byte stores
        for (int x = et; x < nst; x += 128) {
          const int c = x / (nrows * 8), rem = x % (nrows * 8);
          const int t = mt.nt + rem / 8, u = rem % 8;
          *reinterpret_cast<uint4*>(vt + c * 2048 + t * 128 + u * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&pready[s]);
      if (mt.flags & kLast) {
        if (!mbar_wait(zdone, seg & 1)) {
          set_timeout(p.status, kSiteVZdone);
          abort_flag = 1;
          break;
        }
        tc_fence_after();
        const size_t slot = static_cast<size_t>(mt.b) + cta;
        float* zb = p.zpart + (static_cast<size_t>(rr) * p.v_slots + slot) * p.H * p.r_range;
        for (int m = 0; m < p.n_mtiles; ++m) {
          uint32_t v[32];
          const uint32_t ta = taddr + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(m * p.npad);
          const int j = m * 128 + q * 32 + lane;
          for (int h0 = 0; h0 < p.H; h0 += 32) {
            if (p.npad - h0 >= 32) tmem_ld_32x32b_x32(ta + h0, v);
            else tmem_ld_32x32b_x16(ta + h0, v);
            tmem_ld_wait();
            if (j < p.r_range && rr * p.r_range + j < p.R) {
              const int hn = min(32, p.H - h0);
              for (int hh = 0; hh < hn; ++hh)
                zb[static_cast<size_t>(h0 + hh) * p.r_range + j] = __uint_as_float(v[hh]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(tfree);
        // per-segment normaliser of every head
        sRed[et] = lsum;
        named_bar_sync(2, 128);
        if (rr == 0 && et < p.H) {
          float Ls = 0.f;
          for (int i = et; i < 128; i += p.npad) Ls += sRed[i];
          p.lpart[slot * p.H + et] = Ls;
        }
        named_bar_sync(2, 128);
        ++seg;
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(taddr, p.tmem_cols);
  }
}

// ====================================================================== upproj
struct UpProjParams {
  const float* zpart;     // [n_rr][v_slots][H][r_range]
  const float* lpart;     // [v_slots][H]
  const int32_t* prefix;
  const __half* B_V;      // [R][H*d]
  __half* out;            // [B][H][d]
  int B, H, d, R, r_range, v_slots, v_grid;
};

constexpr int kUpBT = 16;   // sequences per CTA
constexpr int kUpRC = 128;  // rows of B_V (and Z) staged per chunk

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// grid (H, ceil(B/16)), 256 threads; dynamic smem 2 x (kUpRC*d halves + kUpRC*16 floats).
// out[b,h,:] = (sum over the V-pass partials of sequence b) . B_V[:, h*d:(h+1)*d]
template <int BPT>
__global__ void __launch_bounds__(256) upproj_kernel(UpProjParams p) {
  extern __shared__ __align__(16) uint8_t up_smem[];
  __half* bvs = reinterpret_cast<__half*>(up_smem);                          // [2][kUpRC][d]
  float* zs = reinterpret_cast<float*>(up_smem + 2 * kUpRC * p.d * 2);       // [2][kUpRC][kUpBT]
  __shared__ int32_t i0s[kUpBT], i1s[kUpBT];
  __shared__ float invl[kUpBT];
  const int h = blockIdx.x;
  const int bt0 = blockIdx.y * kUpBT;
  const int tid = threadIdx.x;
  const int half_d = p.d / 2;
  const int c2 = tid % half_d;
  const int grp = tid / half_d;
  Partition pt;
  pt.P = p.prefix[p.B];
  pt.G = static_cast<int32_t>(pt.P < p.v_grid ? pt.P : p.v_grid);
  if (tid < kUpBT) {
    const int b = bt0 + tid;
    int32_t a = 0, z = -1;
    if (b < p.B && p.prefix[b + 1] > p.prefix[b]) {
      a = part_owner(p.prefix[b], pt);
      z = part_owner(p.prefix[b + 1] - 1, pt);
    }
    i0s[tid] = a;
    i1s[tid] = z;
    float Ls = 0.f;
    for (int32_t i = a; i <= z; ++i) Ls += p.lpart[static_cast<size_t>(b + i) * p.H + h];
    invl[tid] = Ls > 0.f ? 1.f / Ls : 0.f;
  }
  __syncthreads();
  const size_t hd = static_cast<size_t>(p.H) * p.d;
  const int n_chunks = (p.R + kUpRC - 1) / kUpRC;
  const int vec_per_row = p.d / 8;  // 16-byte pieces of one B_V row slice

  auto load_bv = [&](int chunk, int buf) {
    const int j0 = chunk * kUpRC;
    const int jn = min(kUpRC, p.R - j0);
    __half* dst = bvs + static_cast<size_t>(buf) * kUpRC * p.d;
    for (int x = tid; x < jn * vec_per_row; x += 256) {
      const int j = x / vec_per_row, v = x % vec_per_row;
      cp_async16(dst + j * p.d + v * 8, p.B_V + static_cast<size_t>(j0 + j) * hd + static_cast<size_t>(h) * p.d + v * 8);
    }
  };
  auto load_z = [&](int chunk, int buf) {
    const int j0 = chunk * kUpRC;
    const int jn = min(kUpRC, p.R - j0);
    float* dst = zs + static_cast<size_t>(buf) * kUpRC * kUpBT;
    for (int x = tid; x < jn * kUpBT; x += 256) {
      const int bt = x / jn, j = j0 + x % jn;
      const int b = bt0 + bt;
      float z = 0.f;
      if (b < p.B) {
        const int rrg = j / p.r_range, jj = j % p.r_range;
        const float* src = p.zpart + ((static_cast<size_t>(rrg) * p.v_slots + b) * p.H + h) * p.r_range + jj;
        const size_t slot_stride = static_cast<size_t>(p.H) * p.r_range;
        for (int32_t i = i0s[bt]; i <= i1s[bt]; ++i) z += src[static_cast<size_t>(i) * slot_stride];
      }
      dst[(j - j0) * kUpBT + bt] = z;
    }
  };

  float acc[BPT][2];
#pragma unroll
  for (int u = 0; u < BPT; ++u) acc[u][0] = acc[u][1] = 0.f;
  load_bv(0, 0);
  cp_async_commit();
  load_z(0, 0);
  for (int c = 0; c < n_chunks; ++c) {
    const int buf = c & 1;
    if (c + 1 < n_chunks) {
      load_bv(c + 1, buf ^ 1);
      cp_async_commit();
      load_z(c + 1, buf ^ 1);
      cp_async_wait_1();
    } else {
      cp_async_wait_0();
    }
    __syncthreads();
    if (grp * BPT < kUpBT) {
      const int jn = min(kUpRC, p.R - c * kUpRC);
      const __half* bv = bvs + static_cast<size_t>(buf) * kUpRC * p.d + 2 * c2;
      const float* zr0 = zs + static_cast<size_t>(buf) * kUpRC * kUpBT + grp * BPT;
#pragma unroll 4
      for (int j = 0; j < jn; ++j) {
        const float2 w = __half22float2(*reinterpret_cast<const __half2*>(bv + j * p.d));
        const float* zr = zr0 + j * kUpBT;
#pragma unroll
        for (int u = 0; u < BPT; ++u) {
          acc[u][0] = fmaf(zr[u], w.x, acc[u][0]);
          acc[u][1] = fmaf(zr[u], w.y, acc[u][1]);
        }
      }
    }
    __syncthreads();
  }
  if (grp * BPT < kUpBT) {
#pragma unroll
    for (int u = 0; u < BPT; ++u) {
      const int b = bt0 + grp * BPT + u;
      const float il = invl[grp * BPT + u];
      if (b < p.B)
        *reinterpret_cast<__half2*>(p.out + (static_cast<size_t>(b) * p.H + h) * p.d + 2 * c2) =
            __floats2half2_rn(acc[u][0] * il, acc[u][1] * il);
    }
  }
}

}  // namespace starkv
