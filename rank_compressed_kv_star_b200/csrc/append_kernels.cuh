// Compress-and-append: codes of one new token per sequence into the paged pools.
//
// c_K[b,h,:] = k[b,h,:] . A_K[h]  (head-wise K, A_K[h] is d x r)
// c_V[b,:]   = v[b,:] . A_V       (joint V over the concatenated heads, A_V is H*d x R)
// Both are accumulated in fp32, rounded to fp16 (nearest even) and stored in
// slot pos % 16 of page block_table[b][pos / 16] (Proxima README, method
// paragraph: codes "stored in a compressed paged format").
//
// The joint V projection is a dense GEMM over the batch,
//   C_V^T (R x B) = A_V^T (R x H*d) . V^T (H*d x B),
// run on tcgen05 tensor cores: one CTA per (128-row tile of R, K range),
// A tiles are 64x64 boxes of A_V (MN-major, 128B swizzle), B tiles 64-column
// boxes of the batch's v rows (K-major, 128B swizzle), the fp32 accumulator
// lives in tensor memory.  The K ranges of one R tile form a thread-block
// cluster and are summed through distributed shared memory in a fixed order,
// so the result does not depend on scheduling.  The head-wise K codes are
// small per-head products on the CUDA cores.
//
// Both run as tile bodies of the prep kernel (decode_kernels.cuh), which can
// put them in one launch with the decode's query absorption.
#pragma once
#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "../../include/starkv.h"

namespace starkv {

// Where row b's codes go: either an explicit flat slot (page*16 + offset) per
// row, or (block table row, position) per sequence.
struct AppendTarget {
  const int32_t* slots;    // [B] flat slots, or null to use tables/positions
  const int32_t* tables;   // [B][MB]
  const int32_t* positions;
  int MB, NB;
  int32_t* status;         // optional: flags of skipped targets are OR-ed in
};

// Physical row (page*16 + slot) of row b's target, or a negated STARKV_FLAG_*
// naming why the target is skipped: -STARKV_FLAG_BAD_SEQ_LEN for a position
// outside the block table, -STARKV_FLAG_BAD_BLOCK_ID for a page outside the pool.
__device__ __forceinline__ int64_t append_row(const AppendTarget& a, int b) {
  if (a.slots) {
    const int32_t sl = a.slots[b];
    return (sl < 0 || sl >= a.NB * 16) ? -STARKV_FLAG_BAD_BLOCK_ID : static_cast<int64_t>(sl);
  }
  const int32_t pos = a.positions[b];
  if (pos < 0 || pos / 16 >= a.MB) return -STARKV_FLAG_BAD_SEQ_LEN;
  const int32_t phys = a.tables[static_cast<size_t>(b) * a.MB + pos / 16];
  if (phys < 0 || phys >= a.NB) return -STARKV_FLAG_BAD_BLOCK_ID;
  return static_cast<int64_t>(phys) * 16 + (pos % 16);
}

// Records a skipped target (called by one thread per row).
__device__ __forceinline__ void append_skipped(const AppendTarget& a, int64_t why) {
  if (a.status) atomicOr(a.status, static_cast<int32_t>(-why));
}

// ------------------------------------------------------------ V codes (TC)
struct AppendVParams {
  AppendTarget tgt;
  __half* v_cache;         // [NB][16][R]
  int B, HD, R;
  int k_per_cta;           // rows of H*d per CTA (multiple of 64)
  int npad;                // UMMA N: batch tile padded to a multiple of 16 (<= 256)
  int stages;
  uint32_t tmem_cols;
};

constexpr int kPrepThreads = 256;  // threads of every prep-kernel CTA
constexpr int kAppKC = 64;         // rows of H*d per pipeline stage

// One tile of the V-code GEMM: rows [128 mt, 128 mt + 128) of R, the ks-th of
// KS K ranges (the CTA's rank in its (1, KS, 1) cluster), batch tile bt of
// 256 sequences.  Warp 0 issues the TMA copies, warp 1 the MMAs, warps 2..5
// drain the accumulator; all kPrepThreads threads take part in the
// cluster-wide reduction.  `smem` is the 1024-aligned dynamic shared memory.
__device__ __forceinline__ void append_v_tile(const CUtensorMap* amap, const CUtensorMap* vmap,
                                              const AppendVParams& p, int mt, int ks, int KS, int bt,
                                              uint8_t* smem) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int S = p.stages;
  const uint32_t a_bytes = 2u * kAppKC * 128u;                 // two 64x64 fp16 boxes
  const uint32_t b_bytes = static_cast<uint32_t>(p.npad) * 128u;
  const uint32_t stage_bytes = a_bytes + b_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(S) * stage_bytes);
  uint64_t* empty = full + S;
  uint64_t* done = empty + S;
  float* part = reinterpret_cast<float*>(smem);                 // [npad][128], reuses the ring
  __shared__ uint32_t taddr_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b0 = bt * 256;
  const int k0 = ks * p.k_per_cta;
  const int k1 = min(p.HD, k0 + p.k_per_cta);
  const int n_stages = k1 > k0 ? (k1 - k0 + kAppKC - 1) / kAppKC : 0;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(done, 1);
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
  bool ok = true;
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0 && lane == 0) {
    prefetch_tensormap(amap);
    prefetch_tensormap(vmap);
    const uint64_t pol = policy_evict_last();
    for (int i = 0; i < n_stages; ++i) {
      const int s = i % S;
      if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1)) { ok = false; break; }
      uint8_t* st = smem + static_cast<size_t>(s) * stage_bytes;
      const int kr = k0 + i * kAppKC;
      mbar_arrive_expect_tx(&full[s], stage_bytes);
      tma_load_2d(st, amap, mt * 128, kr, &full[s], pol);
      tma_load_2d(st + kAppKC * 128, amap, mt * 128 + 64, kr, &full[s], pol);
      tma_load_2d(st + a_bytes, vmap, kr, b0, &full[s], pol);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_f16_f32(128, p.npad, /*a_mn_major=*/true, /*b_mn_major=*/false);
    for (int i = 0; i < n_stages; ++i) {
      const int s = i % S;
      if (!mbar_wait(&full[s], (i / S) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
      const uint32_t sb = sa + a_bytes;
#pragma unroll
      for (int kk = 0; kk < kAppKC / 16; ++kk) {
        const uint64_t adesc = smem_desc(sa + kk * 16u * 128u, kAppKC * 128u, 1024u, kSwizzle128B);
        const uint64_t bdesc = smem_desc(sb + kk * 32u, 16u, 1024u, kSwizzle128B);
        umma_f16_ss(taddr, adesc, bdesc, idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&empty[s]);
    }
    umma_commit(done);
  }
  __syncthreads();
  // every warp observes the accumulator completion (or an empty K range)
  if (!mbar_wait(done, 0)) ok = false;
  tc_fence_after();
  if (warp >= 2 && warp < 6) {
    const int q = warp & 3;
    const int row = q * 32 + lane;            // row of the R tile
    for (int c0 = 0; c0 < p.npad; c0 += 16) {
      uint32_t v[32];
      tmem_ld_32x32b_x16(taddr + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j)
        part[(c0 + j) * 128 + row] = (n_stages > 0 && ok) ? __uint_as_float(v[j]) : 0.f;
    }
  }
  tc_fence_before();
  cluster.sync();
  // rank ks sums rows (batch entries) [ks*npad/KS, (ks+1)*npad/KS) over the cluster, in rank order
  const int per = (p.npad + KS - 1) / KS;
  const int n_lo = ks * per, n_hi = min(p.npad, n_lo + per);
  // four consecutive rows of R per thread, all ranks' loads issued before the
  // adds (in rank order)
  for (int x = tid; x < (n_hi - n_lo) * 32; x += kPrepThreads) {
    const int n = n_lo + x / 32, rrow = (x % 32) * 4;
    const int b = b0 + n;
    const int rg = mt * 128 + rrow;
    if (b >= p.B || rg >= p.R) continue;
    float4 v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < KS) v[c] = *reinterpret_cast<const float4*>(cluster.map_shared_rank(part, c) + n * 128 + rrow);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < KS) { acc.x += v[c].x; acc.y += v[c].y; acc.z += v[c].z; acc.w += v[c].w; }
    const int64_t dst = append_row(p.tgt, b);
    if (dst >= 0) {
      const __half2 lo = __floats2half2_rn(acc.x, acc.y), hi = __floats2half2_rn(acc.z, acc.w);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(p.v_cache + dst * p.R + rg) = pk;
    } else if (rg == 0) {
      append_skipped(p.tgt, dst);
    }
  }
  cluster.sync();   // nobody leaves while others still read its partials
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(taddr, p.tmem_cols);
  }
}

// ------------------------------------------------------------ small products
// out[b][i] = sum_j x[b][j] * W[j][i] for nb rows of x (fp16 [nb][d]) and W
// (fp16 [d][r]), both staged in shared memory, with fp32 accumulation.
// Thread = (column pair p: columns 2p and 2p+1; row lane bl); each step of 8
// along j it reads 8 column pairs of W (4-byte reads, consecutive across a
// warp) and 8 values of each of up to kProjRows rows (16-byte broadcast
// reads), and accumulates with packed FMAs.  emit(b, i, v_i, v_i+1) receives
// the two columns of row b.  r must be a multiple of 16 (r/2 divides 256).
constexpr int kProjRows = 4;

template <typename Emit>
__device__ __forceinline__ void small_proj(const __half* Ws, const __half* xs, int nb, int d, int r, Emit&& emit) {
  const int np = r >> 1;
  const int nbl = kPrepThreads / np;
  const int p = static_cast<int>(threadIdx.x) % np, bl = static_cast<int>(threadIdx.x) / np;
  for (int b0 = bl; b0 < nb; b0 += nbl * kProjRows) {
    float2 acc[kProjRows];
#pragma unroll
    for (int s = 0; s < kProjRows; ++s) acc[s] = make_float2(0.f, 0.f);
    for (int j = 0; j < d; j += 8) {
      float2 w[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        w[u] = __half22float2(*reinterpret_cast<const __half2*>(Ws + static_cast<size_t>(j + u) * r + 2 * p));
#pragma unroll
      for (int s = 0; s < kProjRows; ++s) {
        const int b = b0 + s * nbl;
        if (b < nb) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xs + static_cast<size_t>(b) * d + j);
          const __half2* x2 = reinterpret_cast<const __half2*>(&xv);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 xf = __half22float2(x2[u]);
            acc[s] = ffma2(make_float2(xf.x, xf.x), w[2 * u], acc[s]);
            acc[s] = ffma2(make_float2(xf.y, xf.y), w[2 * u + 1], acc[s]);
          }
        }
      }
    }
#pragma unroll
    for (int s = 0; s < kProjRows; ++s) {
      const int b = b0 + s * nbl;
      if (b < nb) emit(b, 2 * p, acc[s].x, acc[s].y);
    }
  }
}

// ------------------------------------------------------------ K codes
struct AppendKParams {
  AppendTarget tgt;
  const __half* k;         // [B][H][d]
  const __half* A_K;       // [H][d][r]
  __half* k_cache;         // [NB][16][H][r]
  int B, H, d, r;
  int tile;                // sequences per item (<= kAppKB)
};

// One item: head h, sequences [b0, b0 + tile).  A_K[h] ([d][r]) and the
// tile's k[:, h, :] rows are staged in shared memory (`smem`: d*r + kAppKB*d
// halves) for the small-product routine; codes are stored as fp16 pairs.
constexpr int kAppKB = 32;

__device__ __forceinline__ void append_k_item(const AppendKParams& p, int h, int b0, uint8_t* smem) {
  __half* As = reinterpret_cast<__half*>(smem);                 // [d][r]
  __half* ksm = As + static_cast<size_t>(p.d) * p.r;            // [kAppKB][d]
  const int tid = threadIdx.x;
  const int nb = min(p.tile, p.B - b0);
  const uint4* asrc = reinterpret_cast<const uint4*>(p.A_K + static_cast<size_t>(h) * p.d * p.r);
  for (int x = tid; x < p.d * p.r / 8; x += kPrepThreads) reinterpret_cast<uint4*>(As)[x] = asrc[x];
  for (int x = tid; x < nb * p.d / 8; x += kPrepThreads) {
    const int b = x / (p.d / 8), c = x % (p.d / 8);
    reinterpret_cast<uint4*>(ksm)[x] =
        reinterpret_cast<const uint4*>(p.k + (static_cast<size_t>(b0 + b) * p.H + h) * p.d)[c];
  }
  __syncthreads();
  small_proj(As, ksm, nb, p.d, p.r, [&](int b, int i, float v0, float v1) {
    const int64_t row = append_row(p.tgt, b0 + b);
    if (row >= 0)
      *reinterpret_cast<__half2*>(p.k_cache + (row * p.H + h) * p.r + i) = __floats2half2_rn(v0, v1);
    else if (h == 0 && i == 0) append_skipped(p.tgt, row);
  });
}

}  // namespace starkv
