// Decode kernels of the STAR-KV paged low-rank cache (sm_100a).
//
// One decode is four launches on the caller's stream, each launched with
// programmatic stream serialisation (see griddep_wait):
//   1. absorb      q~ = log2(e)*scale * q . B_K[g(h)]^T; page prefix sums; status
//                  and page-chunk counter reset; per-sequence maxima set to -inf
//   2. kpass       base-2 logits s = q~ . c_K over the K pages, each sequence's
//                  max M merged by float-max atomics (kpass_kernel on CUDA cores
//                  for multi-head attention, taking page chunks from a counter;
//                  kpass_tc_kernel on tcgen05 for grouped queries)
//   3. vpass       Z = sum_t w c_V on tcgen05 tensor cores with w = fp16(exp2(s - M)),
//                  and the normaliser L = sum_t w, per segment
//   4. finish      Z / L summed over the segments and split into fp16 hi + lo,
//                  then out_h = (Z_h / L) . B_V[:, g(h)*d:(g(h)+1)*d] on tcgen05 -> fp16
// with g(h) = h / (H / Hkv) the KV head of query head h (g(h) = h without
// grouping).  A chunked prefill adds prefill_rows_kernel in front: each query
// token of a chunk becomes a decode row of its sequence.
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
#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "append_kernels.cuh"
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

// Float maximum through the integer atomics (ordered bit patterns: max over
// signed ints for v >= 0, min over unsigned for v < 0); works on shared or
// global memory.
__device__ __forceinline__ void atomic_max_f32(float* addr, float v) {
  if (__float_as_int(v) >= 0) atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
  else atomicMin(reinterpret_cast<unsigned int*>(addr), __float_as_uint(v));
}

// Block-table row of decode row b: row b itself, or, for rows that are query
// tokens of a prefill chunk, the row of the sequence row_seq[b].
__device__ __forceinline__ const int32_t* table_row(const int32_t* tables, const int32_t* row_seq, int32_t b, int MB) {
  return tables + static_cast<size_t>(row_seq ? row_seq[b] : b) * MB;
}

// Timeout at pipeline wait `site`: the timeout bit plus a per-site bit (8..15)
// that tells where the pipeline stopped.
enum WaitSite : int32_t {
  kSiteKEmpty = 0, kSiteKFull = 1, kSiteVEmpty = 2, kSiteVPready = 3, kSiteVTfree = 4,
  kSiteVFull = 5, kSiteVZdone = 6, kSiteVMdone = 7
};
__device__ __forceinline__ void set_timeout(int32_t* status, WaitSite site) {
  atomicOr(status, STARKV_FLAG_TIMEOUT | (1 << (8 + site)));
}

// ================================================================ prefill rows
// Rows of a chunked prefill: query token i of sequence b (rows
// row_offsets[b] .. row_offsets[b+1]-1) attends over the sequence's tokens
// 0 .. starts[b] + i, so it is decode row r with the sequence's block table
// and length starts[b] + i + 1.
struct PrefillRowsParams {
  const int32_t* starts;       // [n_seqs] position of each chunk's first token
  const int32_t* row_offsets;  // [n_seqs + 1] first row of each sequence's chunk
  int32_t* row_seq;            // [n_rows] out
  int32_t* row_len;            // [n_rows] out
  int n_seqs, n_rows;
};

__global__ void __launch_bounds__(256) prefill_rows_kernel(PrefillRowsParams p) {
  griddep_wait();
  griddep_launch_dependents();
  const int r = blockIdx.x * 256 + threadIdx.x;
  if (r >= p.n_rows) return;
  int lo = 0, hi = p.n_seqs - 1;     // largest b with row_offsets[b] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.row_offsets[mid] <= r) lo = mid; else hi = mid - 1;
  }
  p.row_seq[r] = lo;
  p.row_len[r] = p.starts[lo] + (r - p.row_offsets[lo]) + 1;
}

// ================================================================ chunk table
// Read-once chunked prefill: the rows of a sequence's chunk are taken nq at a
// time as one virtual sequence whose query heads are the virtual heads
// (h, i) = query head h of the chunk's row i.  Virtual sequence v covers rows
// vs_row0[v] .. + vs_nrows[v] - 1 (consecutive positions starting at
// vs_len[v] - vs_nrows[v]) and attends over tokens [0, vs_len[v]): row i over
// tokens [0, vs_len[v] - vs_nrows[v] + i] (causal).  Entries past the last
// virtual sequence get zero rows and zero length.
struct ChunkTableParams {
  const int32_t* starts;       // [n_seqs] position of each chunk's first token
  const int32_t* row_offsets;  // [n_seqs + 1] first row of each sequence's chunk
  int32_t* vs_seq;             // [nv_max] sequence (block-table row) of each virtual sequence
  int32_t* vs_row0;            // [nv_max]
  int32_t* vs_nrows;           // [nv_max]
  int32_t* vs_len;             // [nv_max]
  int n_seqs, nv_max, log2nq;
};

// one CTA of 256 threads: per-sequence counts, a block-wide scan, the entries
__global__ void __launch_bounds__(256) chunk_table_kernel(ChunkTableParams p) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ int32_t part[16];
  __shared__ int32_t total;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nq = 1 << p.log2nq;
  const int per = (p.n_seqs + 255) / 256;
  const int b0 = tid * per;
  int32_t s = 0;
  for (int b = b0; b < b0 + per && b < p.n_seqs; ++b) {
    const int32_t c = p.row_offsets[b + 1] - p.row_offsets[b];
    s += c > 0 ? (c + nq - 1) >> p.log2nq : 0;
  }
  int32_t v = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) part[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int32_t w = lane < 8 ? part[lane] : 0;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < 8) part[8 + lane] = w;
    if (lane == 7) total = w;
  }
  __syncthreads();
  int32_t at = v - s + (warp > 0 ? part[8 + warp - 1] : 0);
  for (int b = b0; b < b0 + per && b < p.n_seqs; ++b) {
    const int32_t r0 = p.row_offsets[b], c = p.row_offsets[b + 1] - r0;
    for (int32_t js = 0; js * nq < c && at < p.nv_max; ++js, ++at) {
      const int32_t n = min(nq, c - js * nq);
      p.vs_seq[at] = b;
      p.vs_row0[at] = r0 + js * nq;
      p.vs_nrows[at] = n;
      p.vs_len[at] = p.starts[b] + js * nq + n;
    }
  }
  for (int32_t e = total + tid; e < p.nv_max; e += 256) {
    p.vs_seq[e] = 0;
    p.vs_row0[e] = 0;
    p.vs_nrows[e] = 0;
    p.vs_len[e] = 0;
  }
}

// ====================================================================== absorb
struct AbsorbParams {
  const __half* q;        // [B][H][d]
  const __half* B_K;      // [H][r][d]
  const int32_t* seq_lens;
  float* qt;              // [B][H][r]
  __half* qth;            // [B][2H][r]: fp16 q~ (row h) and fp16 of its remainder (row H+h); may be null
  int32_t* prefix;        // [B+1]
  int32_t* teff;          // [B] clamped lengths
  int32_t* status;
  float* mpart_init;      // [n_mpart] set to -inf (maxima merged by atomics later); may be null
  int n_mpart;
  uint32_t* work_ctr;     // the K pass's page-chunk counter, set to 0 by item 0; may be null
  int B, H, d, r, cap;    // cap = min(max_seq_len, max_blocks_per_seq*16)
  int log2G;              // query heads per KV head = 1 << log2G
  float coef;             // scale * log2(e)
  // chunked prefill read once (null vs_row0: decode rows): B counts virtual
  // sequences of 1 << log2nq query rows each, seq_lens are their lengths, and
  // qth is laid out [B][2][H << log2nq][r] with virtual head h * nq + i
  const int32_t* vs_row0; // [B] first query row of each virtual sequence
  const int32_t* vs_nrows;// [B] its rows (0: unused entry)
  int log2nq;
};

// One item: query head h, sequences [b0, b0 + tile) (tile <= kAbsBigTile).  Item 0
// also writes the page prefix sums and resets the status word (every later
// kernel of the decode runs after this one); all items share setting the
// segment-max slots to -inf.  B_K[g(h)] is staged transposed ([d][r]) and the
// tile's q rows as they are, both in shared memory (`smem`: d*r + tile*d
// halves), for the shared small-product routine.
constexpr int kAbsBT = 32;
constexpr int kAbsBigTile = 128;   // rows per absorption item when the absorption runs alone over many rows

__device__ __forceinline__ void absorb_item(const AbsorbParams& p, int item, int n_items, int tile, uint8_t* smem) {
  const int h = item % p.H;
  const int bt0 = (item / p.H) * tile;
  const int tid = threadIdx.x;
  if (item == 0) {
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
    // exclusive scan of the 256 per-thread page counts: warp scans, then the warp totals
    const int lane = tid & 31, warp = tid >> 5;
    int32_t v = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) part[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int32_t w = lane < 8 ? part[lane] : 0;
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < 8) part[8 + lane] = w;       // inclusive totals of warps 0..lane
    }
    __syncthreads();
    int32_t acc = v - s + (warp > 0 ? part[8 + warp - 1] : 0);
    if (tid == 255) {
      p.prefix[p.B] = acc + s;
      *p.status = bad ? STARKV_FLAG_BAD_SEQ_LEN : 0;
      if (p.work_ctr) *p.work_ctr = 0u;
    }
    for (int b = b0; b < b0 + per && b < p.B; ++b) {
      p.prefix[b] = acc;
      acc += (p.teff[b] + kBlock - 1) / kBlock;
    }
  }
  if (p.mpart_init) {
    const int nthr = n_items * 256;
    for (int i = item * 256 + tid; i < p.n_mpart; i += nthr) p.mpart_init[i] = -INFINITY;
  }
  const int D = p.d, r = p.r;
  __half* Ws = reinterpret_cast<__half*>(smem);                 // [d][r]: B_K[g(h)] transposed
  __half* qs = Ws + static_cast<size_t>(D) * r;                 // [tile][d]
  // rows of the item: sequences, or (virtual sequence, row) pairs in chunk mode
  const int n_rows_all = p.vs_row0 ? (p.B << p.log2nq) : p.B;
  const int nb = min(tile, n_rows_all - bt0);
  const __half* bk = p.B_K + static_cast<size_t>(h >> p.log2G) * r * D;   // [r][d]
  for (int x = tid; x < r * (D / 8); x += kPrepThreads) {
    const int i = x % r, jb = x / r;          // consecutive threads: consecutive rank indices
    const uint4 v = *reinterpret_cast<const uint4*>(bk + static_cast<size_t>(i) * D + jb * 8);
    const __half* hv = reinterpret_cast<const __half*>(&v);
#pragma unroll
    for (int u = 0; u < 8; ++u) Ws[(jb * 8 + u) * r + i] = hv[u];
  }
  for (int x = tid; x < nb * (D / 8); x += kPrepThreads) {
    const int bb = x / (D / 8), c = x % (D / 8);
    int64_t qrow = bt0 + bb;
    if (p.vs_row0) {   // row i of virtual sequence v, or a zero row past its chunk
      const int v = (bt0 + bb) >> p.log2nq, i = (bt0 + bb) & ((1 << p.log2nq) - 1);
      qrow = i < p.vs_nrows[v] ? static_cast<int64_t>(p.vs_row0[v]) + i : -1;
    }
    reinterpret_cast<uint4*>(qs)[x] =
        qrow >= 0 ? reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(qrow) * p.H + h) * D)[c]
                  : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  // q~[b,h,i] = coef * sum_j q[b,h,j] * B_K[g(h)][i][j]
  small_proj(Ws, qs, nb, D, r, [&](int bb, int i, float v0, float v1) {
    v0 *= p.coef;
    v1 *= p.coef;
    if (p.vs_row0) {
      // B-operand rows of the read-once K pass: virtual head h * nq + row, hi then lo block
      const int vr = bt0 + bb, v = vr >> p.log2nq, row = vr & ((1 << p.log2nq) - 1);
      const size_t hv = static_cast<size_t>(p.H) << p.log2nq;
      const __half2 hi = __floats2half2_rn(v0, v1);
      const float2 hf = __half22float2(hi);
      __half* dst = p.qth + (static_cast<size_t>(v) * 2 * hv + (static_cast<size_t>(h) << p.log2nq) + row) * r + i;
      *reinterpret_cast<__half2*>(dst) = hi;
      *reinterpret_cast<__half2*>(dst + hv * r) = __floats2half2_rn(v0 - hf.x, v1 - hf.y);
      return;
    }
    const size_t o = (static_cast<size_t>(bt0 + bb) * p.H + h) * r + i;
    *reinterpret_cast<float2*>(p.qt + o) = make_float2(v0, v1);
    if (p.qth) {
      const __half2 hi = __floats2half2_rn(v0, v1);
      const float2 hf = __half22float2(hi);
      __half* row = p.qth + (static_cast<size_t>(bt0 + bb) * 2 * p.H + h) * r + i;
      *reinterpret_cast<__half2*>(row) = hi;
      *reinterpret_cast<__half2*>(row + static_cast<size_t>(p.H) * r) = __floats2half2_rn(v0 - hf.x, v1 - hf.y);
    }
  });
}

// ======================================================================== prep
// One launch for the small per-token work of a step, by CTA role along x
// (clusters of KS CTAs along y):
//   x <  v_cols            tiles of the V-code GEMM of the new tokens (append)
//   x <  v_cols + k_cols   K-code items (head, batch tile) of the new tokens
//   the rest               query-absorption items (head, batch tile) of a decode
// A call runs any subset: the compress-and-append alone (V + K codes), the
// decode's absorption alone, or both at once for a whole step.  The roles read
// and write disjoint data, so they need no order among themselves.
struct PrepParams {
  AppendVParams v;
  AppendKParams k;
  AbsorbParams a;
  int v_mt, v_cols;        // 128-row tiles of R; grid columns of V-code tiles (v_mt * batch tiles)
  int k_items, k_cols;     // K-code items (heads x batch tiles) and their grid columns
  int a_items, a_tile;     // absorption items (heads x batch tiles of a_tile sequences)
};

__global__ void __launch_bounds__(kPrepThreads, 2)
prep_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap vmap, PrepParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int KS = gridDim.y;
  int x = blockIdx.x;
  if (x < p.v_cols) {
    append_v_tile(&amap, &vmap, p.v, x % p.v_mt, blockIdx.y, KS, x / p.v_mt, smem);
    return;
  }
  x -= p.v_cols;
  griddep_wait();
  griddep_launch_dependents();
  if (x < p.k_cols) {
    const int it = x * KS + blockIdx.y;
    if (it < p.k_items) append_k_item(p.k, it % p.k.H, (it / p.k.H) * p.k.tile, smem);
    return;
  }
  x -= p.k_cols;
  const int it = x * KS + blockIdx.y;
  if (it < p.a_items) absorb_item(p.a, it, p.a_items, p.a_tile, smem);
}

// ======================================================================= kpass
struct KPassParams {
  const __half* k_cache;      // [NB][16][H][r]
  const int32_t* tables;      // [B][MB] (or [n_seqs][MB] with row_seq)
  const int32_t* row_seq;     // [B] sequence of each row, or null (row b is sequence b)
  const int32_t* teff;        // [B]
  const int32_t* prefix;      // [B+1]
  const float* qt;            // [B][H][r]
  float* logits;              // [B][t_pad][H]
  float* mpart;               // [B][H]: max of each sequence's base-2 logits (-inf on entry)
  int32_t* status;
  uint32_t* work_ctr;         // next page chunk to hand out (0 on entry)
  int chunk_pages;            // pages per chunk
  int B, H, log2H, r, MB, NB, t_pad;
  int Hkv, log2G;             // KV heads (codes per token) and log2(query heads per KV head)
  int tps;                    // tokens per ring stage (> 16: whole pages of one sequence)
  int stages;
  uint32_t stage_bytes;       // tps*Hkv*r*2
  int drop_stage;             // test hook: this CTA-local stage is never copied (-1: off)
};

constexpr int kKConsumers = 256;            // 8 warps of dot products
constexpr int kKThreads = kKConsumers + 32; // + one producer warp

struct StageMeta { int32_t b, t0, nt, flags; };

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
#ifndef STARKV_K_CTAS_PER_SM
#define STARKV_K_CTAS_PER_SM 1
#endif

template <int L, int CPT>
__global__ void __launch_bounds__(kKThreads, STARKV_K_CTAS_PER_SM) kpass_kernel(KPassParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int S = p.stages;
  uint8_t* ring = smem;
  StageMeta* meta = reinterpret_cast<StageMeta*>(smem + static_cast<size_t>(S) * p.stage_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(meta + S);
  uint64_t* empty = full + S;

  __shared__ volatile int32_t abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kKConsumers / 32); }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();

  if (warp == kKConsumers / 32) {
    // ------------------------------------------------------------ producer
    // Pages are handed out in chunks of chunk_pages from a counter in the
    // workspace, so that a CTA on an SM that streams faster takes more of
    // them (equal static ranges leave the grid waiting for its slowest CTA).
    // The only per-CTA results are the per-sequence maxima, merged by atomics,
    // so which CTA reads a page does not change any result.  A CTA's chunks
    // come in increasing order, so its walk over the sequences only moves on.
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    const uint32_t tok_bytes = static_cast<uint32_t>(p.Hkv) * p.r * 2;
    uint32_t k = 0;
    bool ok = true;
    const int64_t P = p.prefix[p.B];
    const int64_t C = p.chunk_pages;
    const int64_t n_chunks = (P + C - 1) / C;
    const size_t page_elems = static_cast<size_t>(kBlock) * p.Hkv * p.r;
    int32_t b = -1;
    uint32_t c = atomicAdd(p.work_ctr, 1u);
    while (ok && static_cast<int64_t>(c) < n_chunks) {
      const uint32_t c_next = atomicAdd(p.work_ctr, 1u);   // in flight while this chunk is issued
      const int64_t p0 = static_cast<int64_t>(c) * C, p1 = min(P, p0 + C);
      if (b < 0) b = seq_of_page(p.prefix, p.B, p0);
      if (p.tps <= kBlock) {
        // a page is split over several stages
        for (int64_t pg_g = p0; pg_g < p1 && ok; ++pg_g) {
          while (p.prefix[b + 1] <= pg_g) ++b;
          const int32_t pg = static_cast<int32_t>(pg_g - p.prefix[b]);
          const int32_t T = p.teff[b];
          int32_t phys = table_row(p.tables, p.row_seq, b, p.MB)[pg];
          if (phys < 0 || phys >= p.NB) { set_flag(p.status, STARKV_FLAG_BAD_BLOCK_ID); phys = 0; }
          const int32_t tend = min(pg * kBlock + kBlock, T);
          for (int32_t t0 = pg * kBlock; t0 < tend; t0 += p.tps, ++k) {
            const int s = k % S;
            if (k >= static_cast<uint32_t>(S) && !mbar_wait(&empty[s], ((k / S) - 1) & 1)) { ok = false; break; }
            if (static_cast<int>(k) == p.drop_stage) continue;
            const int32_t nt = min(p.tps, tend - t0);
            meta[s] = StageMeta{b, t0, nt, 0};
            const uint32_t bytes = static_cast<uint32_t>(nt) * tok_bytes;
            mbar_arrive_expect_tx(&full[s], bytes);
            const __half* src = p.k_cache + static_cast<size_t>(phys) * page_elems +
                                static_cast<size_t>(t0 - pg * kBlock) * p.Hkv * p.r;
            bulk_g2s(ring + static_cast<size_t>(s) * p.stage_bytes, src, bytes, &full[s], pol);
          }
        }
      } else {
        // a stage gathers up to tps/16 consecutive pages of one sequence, one
        // bulk copy per page, placed back to back (token-major, as in a page)
        const int pps = p.tps / kBlock;
        int64_t pg_g = p0;
        while (pg_g < p1 && ok) {
          while (p.prefix[b + 1] <= pg_g) ++b;
          const int32_t pg = static_cast<int32_t>(pg_g - p.prefix[b]);
          const int32_t T = p.teff[b];
          const int64_t stop = min(p1, static_cast<int64_t>(p.prefix[b + 1]));
          const int n_pg = static_cast<int>(min(static_cast<int64_t>(pps), stop - pg_g));
          const int32_t t0 = pg * kBlock;
          const int32_t nt = min(n_pg * kBlock, T - t0);
          const int s = k % S;
          if (k >= static_cast<uint32_t>(S) && !mbar_wait(&empty[s], ((k / S) - 1) & 1)) { ok = false; break; }
          const bool drop = static_cast<int>(k) == p.drop_stage;
          if (!drop) {
            meta[s] = StageMeta{b, t0, nt, 0};
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nt) * tok_bytes);
          }
          for (int i = 0; i < n_pg && !drop; ++i) {
            int32_t phys = table_row(p.tables, p.row_seq, b, p.MB)[pg + i];
            if (phys < 0 || phys >= p.NB) { set_flag(p.status, STARKV_FLAG_BAD_BLOCK_ID); phys = 0; }
            const int32_t ti = min(kBlock, nt - i * kBlock);
            bulk_g2s(ring + static_cast<size_t>(s) * p.stage_bytes + static_cast<size_t>(i) * kBlock * tok_bytes,
                     p.k_cache + static_cast<size_t>(phys) * page_elems, static_cast<uint32_t>(ti) * tok_bytes,
                     &full[s], pol);
          }
          ++k;
          pg_g += n_pg;
        }
      }
      c = c_next;
    }
    if (ok) {
      const int s = k % S;
      if (k >= static_cast<uint32_t>(S) && !mbar_wait(&empty[s], ((k / S) - 1) & 1)) ok = false;
      if (ok) { meta[s] = StageMeta{-1, 0, 0, 0}; mbar_arrive(&full[s]); }
    }
    if (!ok) {
      set_timeout(p.status, kSiteKEmpty);
      abort_flag = 1;
    }
    // Copies still in flight land before the CTA can exit (consumers that gave
    // up do not wait for them): the last uses of the ring slots, i.e. stages
    // [k - S, k), minus stage k - S when the end marker reused its slot (that
    // stage was consumed, so it had landed).
    const uint32_t first = k >= static_cast<uint32_t>(S) ? k - S + (ok ? 1u : 0u) : 0u;
    for (uint32_t kk = first; kk < k; ++kk) mbar_wait(&full[kk % S], (kk / S) & 1);
    return;
  }

  // -------------------------------------------------------------- consumers
  constexpr int kPairsPerPass = kKConsumers / L;
  constexpr int kRP = CPT <= 4 ? 4 : (CPT <= 8 ? 2 : 1);   // passes held in registers at a time
  const int pair0 = tid / L;
  const int sub = tid % L;
  const int head = pair0 & (p.H - 1);
  const int cp = p.r >> 3;                  // 16-byte chunks per (token, head) row
  const int rot = chunk_rotation(tid, cp, L);
  const int passes = (p.tps * p.H + kPairsPerPass - 1) / kPairsPerPass;
  float2 qv[CPT * 4];
  float m = -INFINITY;
  int cur_b = -1;
  const uint64_t keep = policy_evict_last();   // logits: read back by the V pass

  for (uint32_t k = 0;; ++k) {
    const int s = k % S;
    // warp-uniform decision: the lanes below shuffle with a full mask
    const bool landed = mbar_wait(&full[s], (k / S) & 1);
    if (!__all_sync(0xffffffffu, landed && !abort_flag)) {
      set_timeout(p.status, kSiteKFull);
      break;
    }
    const StageMeta mt = meta[s];
    if (mt.b != cur_b || mt.b < 0) {   // new sequence, or the end marker (b < 0)
      // the sequence's max of every head (-inf on entry), merged across all
      // consumers of all CTAs by float-max atomics
      if (cur_b >= 0 && sub == 0 && m > -INFINITY) atomic_max_f32(&p.mpart[static_cast<size_t>(cur_b) * p.H + head], m);
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
    // The rows of up to kRP passes are copied into registers first; once the
    // last pass's rows are in registers the stage goes back to the producer,
    // so the ring refills while the dot products run (a stage is held only
    // for its shared-memory reads, which keeps more copies in flight).
    const uint8_t* st = ring + static_cast<size_t>(s) * p.stage_bytes;
    for (int ps0 = 0; ps0 < passes; ps0 += kRP) {
      uint4 w[kRP][CPT];
      int tt[kRP];
#pragma unroll
      for (int u = 0; u < kRP; ++u) {
        const int t = ((ps0 + u) * kPairsPerPass + pair0) >> p.log2H;   // token within the stage
        tt[u] = (ps0 + u < passes && t < mt.nt) ? t : -1;
        if (tt[u] >= 0) {
          // code row (token t, KV head of this query head); rows are r*2 bytes
          const uint8_t* row = st + static_cast<size_t>((t << (p.log2H - p.log2G)) + (head >> p.log2G)) * p.r * 2;
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            const int cc = c + rot < CPT ? c + rot : c + rot - CPT;
            const int ch = sub * CPT + cc;
            w[u][c] = ch < cp ? *reinterpret_cast<const uint4*>(row + ch * 16) : make_uint4(0, 0, 0, 0);
          }
        }
      }
      if (ps0 + kRP >= passes) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
#pragma unroll
      for (int u = 0; u < kRP; ++u) {
        float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
        if (tt[u] >= 0) {
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            const __half2* h2 = reinterpret_cast<const __half2*>(&w[u][c]);
            a0 = ffma2(__half22float2(h2[0]), qv[c * 4 + 0], a0);
            a1 = ffma2(__half22float2(h2[1]), qv[c * 4 + 1], a1);
            a2 = ffma2(__half22float2(h2[2]), qv[c * 4 + 2], a2);
            a3 = ffma2(__half22float2(h2[3]), qv[c * 4 + 3], a3);
          }
        }
        float acc = ((a0.x + a0.y) + (a1.x + a1.y)) + ((a2.x + a2.y) + (a3.x + a3.y));
#pragma unroll
        for (int o = L / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (tt[u] >= 0) {
          if (sub == 0)
            st_global_hint(p.logits + (static_cast<size_t>(cur_b) * p.t_pad + mt.t0 + tt[u]) * p.H + head, acc,
                           keep);
          m = fmaxf(m, acc);
        }
      }
    }
  }
}

// ============================================================== kpass (tensor)
// Grouped-query K pass on tcgen05.  With G = H/Hkv query heads per KV head the
// logits of a run of tokens are a small GEMM, S[(t,j), h] = c_K[t, j] . q~_h.
// A tile is 128 code rows: tpt = 128/Hkv tokens of one sequence times the Hkv
// KV heads in page order (row t*Hkv + j), brought in by one 3-D TMA box per
// page {64 codes, Hkv heads, min(16, tpt) tokens} with the 128-byte swizzle,
// which is the K-major operand layout.  B holds the sequence's absorbed
// queries for all H heads split into an fp16 high part (row h) and the fp16
// rounding of the remainder (row H+h); each K step issues one MMA against the
// high rows and one against the low rows into the same accumulator, so
// D[row, h] = c_K . q~_h with q~ carried to about 22 bits and fp32
// accumulation.  B is loaded once per (sequence, CTA) segment into one of nbs
// slots.  A row uses only the G columns of its own KV head; the tensor cores
// compute all H, which at G >= 2 costs less than the HBM time of the tile.
//
// Warp roles: warp 0 (one thread) issues the TMA copies, warp 1 (one thread)
// the MMAs into a ring of nacc TMEM accumulators, warps 2..5 (one TMEM lane
// quarter each) drain them.  Several CTAs share an SM so that the per-tile
// latency chains of different CTAs overlap.  An epilogue warp picks its row's
// G columns, stores them as one contiguous vector (a warp writes whole logit
// rows) and keeps running maxima; at the end of every segment each warp merges
// them into the segment's maxima in global memory (float max through integer
// atomics, initialised to -inf by the absorb kernel).
struct KPassTCParams {
  const int32_t* tables;      // [B][MB] (or [n_seqs][MB] with row_seq)
  const int32_t* row_seq;     // [B] sequence of each row, or null
  const int32_t* teff;        // [B]
  const int32_t* prefix;      // [B+1]
  float* logits;              // [B][t_pad][H]
  float* mpart;               // [B][H]: each sequence's maxima, -inf on entry
  int32_t* status;
  int B, log2G, log2Hkv, MB, NB, t_pad;
  int log2tpt;                // tokens per tile = 128 / Hkv
  int ksteps;                 // UMMA K steps of 16 codes: ceil(r/16)
  int kb;                     // 64-code column blocks: ceil(r/64)
  int nmma;                   // UMMA N = max(16, H): TMEM columns per accumulator
  int brows;                  // rows of a query tile: 2H (H >= 16) or 32
  int nacc;                   // TMEM accumulators (ring)
  int nbs;                    // query-tile slots (1 or 2)
  int stages;
  uint32_t a_bytes;           // kb * 128 rows * 128 bytes
  uint32_t b_bytes;           // kb * brows * 128 bytes
  uint32_t tmem_cols;
  int drop_stage;             // test hook: this CTA-local tile is never copied (-1: off)
};

constexpr int kKTCMaxAcc = 4;
constexpr int kKTCThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue

// Calls f(b, t0, nt, x0, first, last) for the K-pass tiles of pages [p0, p1)
// in order: tokens [t0, t0+nt) of sequence b, whose first token lies in global
// page x0, `first` / `last` on the first and final tile of the (sequence, CTA)
// segment.  Stops when f returns false.
template <typename F>
__device__ __forceinline__ void for_each_k_tile(const KPassTCParams& p, int64_t p0, int64_t p1, F&& f) {
  const int tpt = 1 << p.log2tpt;
  int32_t b = seq_of_page(p.prefix, p.B, p0);
  int64_t x = p0;
  while (x < p1) {
    while (p.prefix[b + 1] <= x) ++b;
    const int64_t seg_end = min(p1, static_cast<int64_t>(p.prefix[b + 1]));
    const int32_t base = p.prefix[b];
    const int32_t ts = static_cast<int32_t>(x - base) * kBlock;
    const int32_t te = min(static_cast<int32_t>(seg_end - base) * kBlock, p.teff[b]);
    for (int32_t t0 = ts; t0 < te; t0 += tpt)
      if (!f(b, t0, min(tpt, te - t0), static_cast<int64_t>(base) + (t0 >> 4), t0 == ts, t0 + tpt >= te)) return;
    x = seg_end;
  }
}

template <int G, int H>   // query heads per KV head, query heads
__global__ void __launch_bounds__(kKTCThreads, 1)
kpass_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                KPassTCParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int S = p.stages;
  uint8_t* bslot = smem + static_cast<size_t>(S) * p.a_bytes;                    // [nbs] query tiles
  uint64_t* full = reinterpret_cast<uint64_t*>(bslot + p.nbs * static_cast<size_t>(p.b_bytes));
  uint64_t* empty = full + S;
  uint64_t* bfull = empty + S;                     // [2] query tile landed
  uint64_t* bempty = bfull + 2;                    // [2] query tile no longer read
  uint64_t* tfull = bempty + 2;                    // [kKTCMaxAcc] accumulator ready
  uint64_t* tempty = tfull + kKTCMaxAcc;           // [kKTCMaxAcc] accumulator drained
  uint64_t* mmadone = tempty + kKTCMaxAcc;         // every MMA issued has completed
  __shared__ uint32_t taddr_s;
  __shared__ volatile int32_t abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&bfull[a], 1); mbar_init(&bempty[a], 1); }
    for (int a = 0; a < kKTCMaxAcc; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 4); }
    mbar_init(mmadone, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  griddep_wait();
  griddep_launch_dependents();
  Partition pt;
  pt.P = p.prefix[p.B];
  pt.G = static_cast<int32_t>(pt.P < gridDim.x ? pt.P : gridDim.x);
  const int cta = blockIdx.x;
  if (cta >= pt.G) return;   // uniform over the CTA
  if (warp == 1) {
    tmem_alloc(&taddr_s, p.tmem_cols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = taddr_s;
  const int64_t p0 = part_begin(cta, pt), p1 = part_begin(cta + 1, pt);
  const int tpt = 1 << p.log2tpt;
  const int Hkv = 1 << p.log2Hkv;
  const int tb = tpt < kBlock ? tpt : kBlock;       // tokens per TMA box (one page, or half of one)

  // Ring positions are advanced incrementally (no divisions per tile): a ring
  // of n slots at position (i, u) is slot i in its u-th use.
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&qmap);
      const uint64_t stream = policy_evict_first();
      const uint64_t reuse = policy_evict_last();
      const uint32_t box_bytes = static_cast<uint32_t>(tb) * Hkv * 128u;
      const int log2tb = tpt < kBlock ? p.log2tpt : 4;
      int si = 0, bi = 0;
      uint32_t su = 0, bu = 0, issued = 0;
      int32_t bpar[2] = {-1, -1};   // parity of each query slot's latest load (-1: none)
      bool ok = true;
      for_each_k_tile(p, p0, p1, [&](int32_t b, int32_t t0, int32_t nt, int64_t x0, bool first, bool last) {
        if (first) {
          if (bu > 0 && !mbar_wait(&bempty[bi], (bu - 1) & 1)) { ok = false; return false; }
          bpar[bi] = static_cast<int32_t>(bu & 1);
          mbar_arrive_expect_tx(&bfull[bi], p.b_bytes);
          for (int a = 0; a < p.kb; ++a)
            tma_load_2d(bslot + bi * static_cast<size_t>(p.b_bytes) + static_cast<size_t>(a) * p.brows * 128, &qmap,
                        a * 64, b * 2 * H, &bfull[bi], reuse);
        }
        if (su > 0 && !mbar_wait(&empty[si], (su - 1) & 1)) { ok = false; return false; }
        uint8_t* st = smem + static_cast<size_t>(si) * p.a_bytes;
        const bool drop = static_cast<int>(issued) == p.drop_stage;
        const int nbox = drop ? 0 : (nt + tb - 1) >> log2tb;
        if (!drop) mbar_arrive_expect_tx(&full[si], static_cast<uint32_t>(nbox * p.kb) * box_bytes);
        const int32_t* trow = table_row(p.tables, p.row_seq, b, p.MB);
        for (int c = 0; c < nbox; ++c) {
          const int32_t t = t0 + c * tb;
          int32_t phys = trow[t >> 4];
          if (phys < 0 || phys >= p.NB) { set_flag(p.status, STARKV_FLAG_BAD_BLOCK_ID); phys = 0; }
          const int32_t row = phys * kBlock + (t & (kBlock - 1));
          for (int a = 0; a < p.kb; ++a)
            tma_load_3d(st + static_cast<size_t>(a) * 16384 + static_cast<size_t>(c) * box_bytes, &kmap, a * 64, 0,
                        row, &full[si], stream);
        }
        ++issued;
        if (++si == S) { si = 0; ++su; }
        if (last && ++bi == p.nbs) { bi = 0; ++bu; }
        return true;
      });
      if (!ok) {
        set_timeout(p.status, kSiteKEmpty);
        abort_flag = 1;
      }
      // copies still in flight land before the CTA can exit (the MMA and
      // epilogue warps may have given up): the last min(issued, S) stages and
      // the latest load of each query slot
      int i = si;
      uint32_t u = su;
      for (uint32_t n = 0; n < issued && n < static_cast<uint32_t>(S); ++n) {
        if (--i < 0) { i = S - 1; --u; }
        mbar_wait(&full[i], u & 1);
      }
      for (int a = 0; a < 2; ++a)
        if (bpar[a] >= 0) mbar_wait(&bfull[a], static_cast<uint32_t>(bpar[a]));
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    // The query slot is released by a commit at every segment end.
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, p.nmma, /*a_mn_major=*/false, /*b_mn_major=*/false);
      const uint32_t b_atom = static_cast<uint32_t>(p.brows) * 8u;    // brows * 128 bytes >> 4
      int si = 0, bi = 0, ai = 0;
      uint32_t su = 0, bu = 0, au = 0;
      bool ok = true;
      for_each_k_tile(p, p0, p1, [&](int32_t, int32_t, int32_t, int64_t, bool, bool last) {
        if (!mbar_wait(&bfull[bi], bu & 1)) { ok = false; return false; }
        if (au > 0 && !mbar_wait(&tempty[ai], (au - 1) & 1)) { ok = false; return false; }
        if (!mbar_wait(&full[si], su & 1) || abort_flag) { ok = false; return false; }
        tc_fence_after();
        // descriptors of the stage / query slot; a K step adds its byte offset >> 4 to the start field
        const uint64_t da = smem_desc(smem_u32(smem + static_cast<size_t>(si) * p.a_bytes), 16u, 1024u, kSwizzle128B);
        const uint64_t db = smem_desc(smem_u32(bslot + bi * static_cast<size_t>(p.b_bytes)), 16u, 1024u, kSwizzle128B);
        const uint32_t d = taddr + static_cast<uint32_t>(ai * p.nmma);
        for (int ks = 0; ks < p.ksteps; ++ks) {
          const uint32_t a = ks >> 2, kk = ks & 3;
          const uint64_t dak = da + (a * 1024u + kk * 2u), dbk = db + (a * b_atom + kk * 2u);
          umma_f16_ss(d, dak, dbk, idesc, ks > 0 ? 1u : 0u);                    // high parts (rows 0..)
          umma_f16_ss(d, dak, dbk + static_cast<uint32_t>(H) * 8u, idesc, 1u);  // low parts (rows H..)
        }
        umma_commit(&empty[si]);
        umma_commit(&tfull[ai]);
        if (++ai == p.nacc) { ai = 0; ++au; }
        if (last) {
          umma_commit(&bempty[bi]);
          if (++bi == p.nbs) { bi = 0; ++bu; }
        }
        if (++si == S) { si = 0; ++su; }
        return true;
      });
      if (!ok) { set_timeout(p.status, kSiteKFull); abort_flag = 1; }
      umma_commit(mmadone);
      mbar_wait(mmadone, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Row rho of a tile is token rho / Hkv, KV head j = rho % Hkv; the row's
    // logits are accumulator columns [j*G, j*G + G).
    const int q = warp & 3;                          // TMEM lane quarter of this warp
    const int rho = q * 32 + lane;
    const int j = rho & (Hkv - 1);
    const int tl = rho >> p.log2Hkv;
    const uint64_t keep = policy_evict_last();       // logits: read back by the V pass
    const uint32_t tq = taddr + (static_cast<uint32_t>(q * 32) << 16);
    float m[G];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) m[gg] = -INFINITY;
    int ai = 0;
    uint32_t au = 0;
    bool ok = true;
    for_each_k_tile(p, p0, p1, [&](int32_t b, int32_t t0, int32_t nt, int64_t, bool, bool last) {
      {
        // warp-uniform decision: the TMEM loads below are .sync.aligned
        const bool ready = mbar_wait(&tfull[ai], au & 1);
        if (!__all_sync(0xffffffffu, ready && !abort_flag)) { ok = false; return false; }
        tc_fence_after();
        const uint32_t tbase = tq + static_cast<uint32_t>(ai * p.nmma);
        float o[G];
        if constexpr (H >= 32) {
          // all loads of the row's H columns in flight before a single wait
          uint32_t v0[32], v1[32];
          tmem_ld_32x32b_x32(tbase, v0);
          if constexpr (H == 64) tmem_ld_32x32b_x32(tbase + 32, v1);
          tmem_ld_wait();
#pragma unroll
          for (int col = 0; col < H; ++col)
            if ((col / G) == j) o[col % G] = __uint_as_float(col < 32 ? v0[col] : v1[col - 32]);
        } else {
          uint32_t v[32];
          tmem_ld_32x32b_x16(tbase, v);             // H <= 16 heads: one 16-column load
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (c < H && (c / G) == j) o[c % G] = __uint_as_float(v[c]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[ai]);
        if (++ai == p.nacc) { ai = 0; ++au; }
        if (tl < nt) {
          float* lrow = p.logits + (static_cast<size_t>(b) * p.t_pad + t0 + tl) * H + j * G;
#pragma unroll
          for (int gg = 0; gg < G; ++gg) m[gg] = fmaxf(m[gg], o[gg]);
          if constexpr (G >= 4) {
#pragma unroll
            for (int gg = 0; gg < G; gg += 4)
              st_global_hint(reinterpret_cast<float4*>(lrow + gg), make_float4(o[gg], o[gg + 1], o[gg + 2], o[gg + 3]),
                             keep);
          } else {
            st_global_hint(reinterpret_cast<uint2*>(lrow), make_uint2(__float_as_uint(o[0]), __float_as_uint(o[1])),
                           keep);
          }
        }
      }
      if (last) {
        // this warp's maxima of the segment (all of its tiles precede this one in the walk)
        float* mp = p.mpart + static_cast<size_t>(b) * H;   // the sequence's maxima
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const float w = warp_max_f32((h / G) == j ? m[h % G] : -INFINITY);
          if (lane == 0 && w > -INFINITY) atomic_max_f32(mp + h, w);
        }
#pragma unroll
        for (int gg = 0; gg < G; ++gg) m[gg] = -INFINITY;
      }
      return true;
    });
    if (!ok) set_timeout(p.status, kSiteKFull);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(taddr, p.tmem_cols);
  }
}

// ============================================================ kpass (chunks)
// Read-once K pass of a chunked prefill on tcgen05.  The virtual heads (h, i)
// of a virtual sequence (query head h of its chunk row i) that share KV head
// g(h) share its K codes: VPK = G x nq of them per KV head, with nq = 16 rows
// per virtual sequence for G <= 4 (a 16-row chunk is one virtual sequence and
// every page is read once) and VPK = 64 above (nq = 64 / G).  A tile is 128
// rows (token, KV head) of KVT KV heads: one page of 8 KV heads (VPK <= 32),
// or two pages of 4 KV heads (VPK = 64), one 3-D TMA box {64 codes, KVT
// heads, 16 tokens} per page and 64 codes; B holds the KVT x VPK virtual heads
// of the group (rows: fp16 high parts, then the low parts), loaded once per
// (segment, group), and the MMA has N = KVT x VPK (128 or 256).  A CTA walks
// each virtual sequence of its page range once per group.  An epilogue lane
// owns one row: it keeps its KV head's VPK columns, sets logits past the
// row's causal limit or the sequence end to -inf, stores them as consecutive
// logits and keeps running maxima that are merged into the segment slots
// (float max) at the end of each pass.
struct KPassChunkParams {
  const int32_t* tables;      // [n_seqs][MB]
  const int32_t* vs_seq;      // [B] sequence of each virtual sequence
  const int32_t* vs_nrows;    // [B] rows of each virtual sequence
  const int32_t* teff;        // [B] lengths
  const int32_t* prefix;      // [B+1]
  float* logits;              // [B][n_vg][t_pad][lw]
  float* mpart;               // [k_slots][Hv], -inf on entry
  int32_t* status;
  int B, MB, NB, t_pad;
  int Hv, n_vg, log2lw;       // virtual heads, groups of lw of them (lw >= VPK)
  int n_groups;               // KV-head groups of KVT
  int log2nq;
  int ksteps, kb;             // UMMA K steps of 16 codes; 64-code column blocks
  int nacc, nbs, stages;
  uint32_t a_bytes;           // kb * 16 KiB
  uint32_t b_bytes;           // kb * 2 * N rows * 128 B
  uint32_t tmem_cols;
  int drop_stage;             // test hook (-1: off)
};

// Tile geometry for VPK virtual heads per KV head.
template <int VPK>
struct ChunkTile {
  static constexpr int kKvt = VPK >= 64 ? 4 : 8;    // KV heads per tile
  static constexpr int kCols = kKvt * VPK;           // UMMA N (128 or 256)
  static constexpr int kTokens = 128 / kKvt;          // tokens per tile (16 or 32)
  static constexpr int kPages = kTokens / kBlock;    // pages per tile (1 or 2)
};

// Calls f(v, pg, np, nt, g, first, last) for the tiles of pages [p0, p1): np
// (<= ppt) consecutive pages from page pg of virtual sequence v (tokens [16 pg,
// 16 pg + nt)) for KV-head group g, each (v, g) pass over the CTA's pages of
// v in page order, `first` / `last` on the pass's first and final tile.  Stops
// when f returns false.
template <typename F>
__device__ __forceinline__ void for_each_chunk_tile(const KPassChunkParams& p, int64_t p0, int64_t p1, int ppt,
                                                    F&& f) {
  int32_t v = seq_of_page(p.prefix, p.B, p0);
  int64_t x = p0;
  while (x < p1) {
    while (p.prefix[v + 1] <= x) ++v;
    const int64_t seg_end = min(p1, static_cast<int64_t>(p.prefix[v + 1]));
    const int32_t base = p.prefix[v];
    const int32_t T = p.teff[v];
    for (int g = 0; g < p.n_groups; ++g)
      for (int64_t y = x; y < seg_end; y += ppt) {
        const int32_t pg = static_cast<int32_t>(y - base);
        const int np = static_cast<int>(min(static_cast<int64_t>(ppt), seg_end - y));
        if (!f(v, pg, np, min(np * kBlock, T - pg * kBlock), g, y == x, y + ppt >= seg_end)) return;
      }
    x = seg_end;
  }
}

template <int VPK>
__global__ void __launch_bounds__(kKTCThreads, 1)
kpass_chunk_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                   KPassChunkParams p) {
  using Geo = ChunkTile<VPK>;
  constexpr int KVT = Geo::kKvt, NCOL = Geo::kCols, PPT = Geo::kPages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int S = p.stages;
  uint8_t* bslot = smem + static_cast<size_t>(S) * p.a_bytes;                    // [nbs] query tiles
  uint64_t* full = reinterpret_cast<uint64_t*>(bslot + p.nbs * static_cast<size_t>(p.b_bytes));
  uint64_t* empty = full + S;
  uint64_t* bfull = empty + S;
  uint64_t* bempty = bfull + 2;
  uint64_t* tfull = bempty + 2;
  uint64_t* tempty = tfull + kKTCMaxAcc;
  uint64_t* mmadone = tempty + kKTCMaxAcc;
  __shared__ uint32_t taddr_s;
  __shared__ volatile int32_t abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&bfull[a], 1); mbar_init(&bempty[a], 1); }
    for (int a = 0; a < kKTCMaxAcc; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 4); }
    mbar_init(mmadone, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  griddep_wait();
  griddep_launch_dependents();
  Partition pt;
  pt.P = p.prefix[p.B];
  pt.G = static_cast<int32_t>(pt.P < gridDim.x ? pt.P : gridDim.x);
  const int cta = blockIdx.x;
  if (cta >= pt.G) return;   // uniform over the CTA
  if (warp == 1) {
    tmem_alloc(&taddr_s, p.tmem_cols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = taddr_s;
  const int64_t p0 = part_begin(cta, pt), p1 = part_begin(cta + 1, pt);
  const int nq1 = (1 << p.log2nq) - 1;
  constexpr uint32_t kBoxBytes = static_cast<uint32_t>(KVT) * kBlock * 128u;   // one page of KVT heads, 64 codes

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&qmap);
      const uint64_t stream = policy_evict_first();
      const uint64_t reuse = policy_evict_last();
      int si = 0, bi = 0;
      uint32_t su = 0, bu = 0, issued = 0;
      int32_t bpar[2] = {-1, -1};
      bool ok = true;
      for_each_chunk_tile(p, p0, p1, PPT, [&](int32_t v, int32_t pg, int np, int32_t, int g, bool first, bool last) {
        if (first) {
          if (bu > 0 && !mbar_wait(&bempty[bi], (bu - 1) & 1)) { ok = false; return false; }
          bpar[bi] = static_cast<int32_t>(bu & 1);
          mbar_arrive_expect_tx(&bfull[bi], p.b_bytes);
          const int hi_row = v * 2 * p.Hv + g * NCOL;
          for (int a = 0; a < p.kb; ++a) {
            uint8_t* dst = bslot + bi * static_cast<size_t>(p.b_bytes) + static_cast<size_t>(a) * 2 * NCOL * 128;
            tma_load_2d(dst, &qmap, a * 64, hi_row, &bfull[bi], reuse);
            tma_load_2d(dst + NCOL * 128, &qmap, a * 64, hi_row + p.Hv, &bfull[bi], reuse);
          }
        }
        if (su > 0 && !mbar_wait(&empty[si], (su - 1) & 1)) { ok = false; return false; }
        uint8_t* st = smem + static_cast<size_t>(si) * p.a_bytes;
        const bool drop = static_cast<int>(issued) == p.drop_stage;
        if (!drop) {
          mbar_arrive_expect_tx(&full[si], static_cast<uint32_t>(np * p.kb) * kBoxBytes);
          const int32_t* trow = table_row(p.tables, p.vs_seq, v, p.MB);
          for (int pp = 0; pp < np; ++pp) {
            int32_t phys = trow[pg + pp];
            if (phys < 0 || phys >= p.NB) { set_flag(p.status, STARKV_FLAG_BAD_BLOCK_ID); phys = 0; }
            for (int a = 0; a < p.kb; ++a)
              tma_load_3d(st + static_cast<size_t>(a) * 16384 + static_cast<size_t>(pp) * kBoxBytes, &kmap, a * 64,
                          g * KVT, phys * kBlock, &full[si], stream);
          }
        }
        ++issued;
        if (++si == S) { si = 0; ++su; }
        if (last && ++bi == p.nbs) { bi = 0; ++bu; }
        return true;
      });
      if (!ok) {
        set_timeout(p.status, kSiteKEmpty);
        abort_flag = 1;
      }
      int i = si;
      uint32_t u = su;
      for (uint32_t n = 0; n < issued && n < static_cast<uint32_t>(S); ++n) {
        if (--i < 0) { i = S - 1; --u; }
        mbar_wait(&full[i], u & 1);
      }
      for (int a = 0; a < 2; ++a)
        if (bpar[a] >= 0) mbar_wait(&bfull[a], static_cast<uint32_t>(bpar[a]));
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, NCOL, /*a_mn_major=*/false, /*b_mn_major=*/false);
      const uint32_t b_atom = 2u * NCOL * 8u;   // one 64-code block of B: 2N rows * 128 bytes >> 4
      int si = 0, bi = 0, ai = 0;
      uint32_t su = 0, bu = 0, au = 0;
      bool ok = true;
      for_each_chunk_tile(p, p0, p1, PPT, [&](int32_t, int32_t, int, int32_t, int, bool, bool last) {
        if (!mbar_wait(&bfull[bi], bu & 1)) { ok = false; return false; }
        if (au > 0 && !mbar_wait(&tempty[ai], (au - 1) & 1)) { ok = false; return false; }
        if (!mbar_wait(&full[si], su & 1) || abort_flag) { ok = false; return false; }
        tc_fence_after();
        const uint64_t da = smem_desc(smem_u32(smem + static_cast<size_t>(si) * p.a_bytes), 16u, 1024u, kSwizzle128B);
        const uint64_t db = smem_desc(smem_u32(bslot + bi * static_cast<size_t>(p.b_bytes)), 16u, 1024u, kSwizzle128B);
        const uint32_t d = taddr + static_cast<uint32_t>(ai * NCOL);
        for (int ks = 0; ks < p.ksteps; ++ks) {
          const uint32_t a = ks >> 2, kk = ks & 3;
          const uint64_t dak = da + (a * 1024u + kk * 2u), dbk = db + (a * b_atom + kk * 2u);
          umma_f16_ss(d, dak, dbk, idesc, ks > 0 ? 1u : 0u);                       // high parts
          umma_f16_ss(d, dak, dbk + static_cast<uint32_t>(NCOL) * 8u, idesc, 1u);  // low parts
        }
        umma_commit(&empty[si]);
        umma_commit(&tfull[ai]);
        if (++ai == p.nacc) { ai = 0; ++au; }
        if (last) {
          umma_commit(&bempty[bi]);
          if (++bi == p.nbs) { bi = 0; ++bu; }
        }
        if (++si == S) { si = 0; ++su; }
        return true;
      });
      if (!ok) { set_timeout(p.status, kSiteKFull); abort_flag = 1; }
      umma_commit(mmadone);
      mbar_wait(mmadone, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp quarter q holds tile rows 32q..32q+31; lane L: row 32q + L = token
    // (32q + L) / KVT of the tile, KV head (L % KVT) of the group, whose
    // columns are [VPK j, VPK j + VPK)
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const int jl = row % KVT;
    const int t = row / KVT;
    const uint64_t keep = policy_evict_last();       // logits: read back by the V pass
    const uint32_t tq = taddr + (static_cast<uint32_t>(q * 32) << 16);
    float m[VPK];
#pragma unroll
    for (int c = 0; c < VPK; ++c) m[c] = -INFINITY;
    int ai = 0;
    uint32_t au = 0;
    bool ok = true;
    for_each_chunk_tile(p, p0, p1, PPT, [&](int32_t v, int32_t pg, int, int32_t nt, int g, bool, bool last) {
      const bool ready = mbar_wait(&tfull[ai], au & 1);
      if (!__all_sync(0xffffffffu, ready && !abort_flag)) { ok = false; return false; }
      tc_fence_after();
      float xs[VPK];
#pragma unroll
      for (int cb = 0; cb < NCOL / 32; ++cb) {   // columns 32 cb .. 32 cb + 31
        uint32_t w[32];
        tmem_ld_32x32b_x32(tq + static_cast<uint32_t>(ai * NCOL + 32 * cb), w);
        tmem_ld_wait();
        if constexpr (VPK == 16) {             // two KV heads per block
          if ((jl >> 1) == cb) {
#pragma unroll
            for (int c = 0; c < 16; ++c) xs[c] = __uint_as_float((jl & 1) ? w[16 + c] : w[c]);
          }
        } else {                               // VPK / 32 blocks per KV head
          if (jl == cb / (VPK / 32)) {
#pragma unroll
            for (int c = 0; c < 32; ++c) xs[(cb % (VPK / 32)) * 32 + c] = __uint_as_float(w[c]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ai]);
      if (++ai == p.nacc) { ai = 0; ++au; }
      {
        // every token slot of the tile's pages gets a logit: -inf past the
        // sequence end too
        const int32_t tabs = pg * kBlock + t;
        const int32_t nrows = p.vs_nrows[v];
        const int32_t rel = tabs - (p.teff[v] - nrows);   // rows i >= rel see this token
        float o[VPK];
#pragma unroll
        for (int c = 0; c < VPK; ++c) {
          const int i = c & nq1;
          o[c] = (t < nt && i < nrows && i >= rel) ? xs[c] : -INFINITY;
          m[c] = fmaxf(m[c], o[c]);
        }
        if (t < ((nt + kBlock - 1) & ~(kBlock - 1))) {   // tokens of pages this tile loaded
          const int vh = g * NCOL + jl * VPK;            // VPK consecutive virtual heads, in one group
          const size_t lrow_idx = (static_cast<size_t>(v) * p.n_vg + (vh >> p.log2lw)) * p.t_pad + tabs;
          float* lrow = p.logits + (lrow_idx << p.log2lw) + (vh & ((1 << p.log2lw) - 1));
#pragma unroll
          for (int c = 0; c < VPK; c += 4)
            st_global_hint(reinterpret_cast<float4*>(lrow + c), make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]),
                           keep);
        }
      }
      if (last) {
        // the maxima of this (segment, group) pass over the warp's rows of each KV head
#pragma unroll
        for (int c = 0; c < VPK; ++c) {
          float x = m[c];
#pragma unroll
          for (int o2 = KVT; o2 < 32; o2 <<= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o2));
          m[c] = x;
        }
        if (lane < KVT) {
          float* mp = p.mpart + static_cast<size_t>(v + cta) * p.Hv + g * NCOL + jl * VPK;
#pragma unroll
          for (int c = 0; c < VPK; ++c)
            if (m[c] > -INFINITY) atomic_max_f32(mp + c, m[c]);
        }
#pragma unroll
        for (int c = 0; c < VPK; ++c) m[c] = -INFINITY;
      }
      return true;
    });
    if (!ok) set_timeout(p.status, kSiteKFull);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(taddr, p.tmem_cols);
  }
}

// ============================================================ chunk weights
// Read-once chunked prefill, between the K and V passes: the attention
// weights of every virtual head, once.  CTA (v, pc, vg) owns pages
// [pc * kCwPages, (pc + 1) * kCwPages) of virtual sequence v for the lw
// virtual heads of group vg.  M = the max over the K pass's segments of v;
// w = fp16(exp2(s - M)) (0 for a logit of -inf: past the row's causal limit,
// or no row).  A page's 16 x lw weights go, in the V pass's B-operand layout
// (K-major core matrices of 8 tokens x 8 heads, i.e. halves [t / 8][head][t %
// 8]), to the page's tile of wts.  The normaliser partial
// of the CTA (the rounded weights summed per page lane in token order, then
// over the page lanes in order) goes to lwpart[v][pc][Hv].
constexpr int kCwPages = 32;
struct ChunkWeightsParams {
  const float* logits;        // [B][n_vg][t_pad][lw]
  __half* wts;                // [B][n_vg][t_pad][lw] fp16: each page's 16 x lw tile in the B-operand layout
  const float* mpart;         // [k_slots][Hv]
  const int32_t* teff;        // [B]
  const int32_t* prefix;      // [B+1]
  float* lwpart;              // [B][n_pc][Hv]: per page chunk sums of the weights of each virtual head
  int B, Hv, n_vg, lw, log2lw, t_pad, k_grid, n_pc;
};

// Thread = (page lane, 4 consecutive virtual heads): 16 float4 loads take a
// page's logits of its heads, and 8 16-byte stores write their weights.
// Hv is a multiple of lw (both powers of two), so every head is live; the K
// pass wrote -inf for every logit that has no weight (past a row's causal
// limit or the sequence end), and ex2 of -inf is exactly 0.
__global__ void __launch_bounds__(256) chunk_weights_kernel(ChunkWeightsParams p) {
  __shared__ float4 sL[256];
  griddep_wait();
  griddep_launch_dependents();
  const int v = blockIdx.x, pc = blockIdx.y, vg = blockIdx.z, tid = threadIdx.x;
  const int log2tpp = p.log2lw - 2;                 // threads per page: lw / 4
  const int c4 = tid & ((1 << log2tpp) - 1), lane_pg = tid >> log2tpp;
  const int gp = 256 >> log2tpp;                    // pages handled side by side
  const int32_t T = p.teff[v];
  const int n_pages = T > 0 ? (T + kBlock - 1) / kBlock : 0;
  const int pg0 = pc * kCwPages, pg1 = min(n_pages, pg0 + kCwPages);   // uniform over the CTA
  const int hcol = vg * p.lw + 4 * c4;
  float M[4] = {0.f, 0.f, 0.f, 0.f};
  if (pg0 < pg1) {
    Partition ptk;
    ptk.P = p.prefix[p.B];
    ptk.G = static_cast<int32_t>(ptk.P < p.k_grid ? ptk.P : p.k_grid);
    const int32_t i0 = part_owner(p.prefix[v], ptk), i1 = part_owner(p.prefix[v + 1] - 1, ptk);
    float4 m = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    for (int32_t i = i0; i <= i1; ++i) {
      const float4 x = *reinterpret_cast<const float4*>(p.mpart + static_cast<size_t>(v + i) * p.Hv + hcol);
      m = make_float4(fmaxf(m.x, x.x), fmaxf(m.y, x.y), fmaxf(m.z, x.z), fmaxf(m.w, x.w));
    }
    // a head with no visible token keeps M = 0: all its logits are -inf
    M[0] = m.x > -INFINITY ? m.x : 0.f;
    M[1] = m.y > -INFINITY ? m.y : 0.f;
    M[2] = m.z > -INFINITY ? m.z : 0.f;
    M[3] = m.w > -INFINITY ? m.w : 0.f;
  }
  const size_t seq_off = (static_cast<size_t>(v) * p.n_vg + vg) * p.t_pad * p.lw;
  const float* seq_logits = p.logits + seq_off;
  __half* seq_wts = p.wts + seq_off;
  const int row4 = p.lw >> 2;                       // float4 per token row
  float L[4] = {0.f, 0.f, 0.f, 0.f};
  for (int pgb = pg0; pgb < pg1; pgb += gp) {
    const int pg = pgb + lane_pg;
    const bool have = pg < pg1;
    const float4* lt = reinterpret_cast<const float4*>(seq_logits + static_cast<size_t>(pg) * kBlock * p.lw) + c4;
    float4 x[kBlock];
#pragma unroll
    for (int t = 0; t < kBlock; ++t)
      x[t] = have ? lt[t * row4] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    if (have) {
      uint32_t w[4][kBlock / 2];
#pragma unroll
      for (int t2 = 0; t2 < kBlock / 2; ++t2) {
        const float4 a = x[2 * t2], b = x[2 * t2 + 1];
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2 h = __floats2half2_rn(ex2_approx(av[j] - M[j]), ex2_approx(bv[j] - M[j]));
          const float2 f = __half22float2(h);
          L[j] += f.x;
          L[j] += f.y;
          w[j][t2] = *reinterpret_cast<const uint32_t*>(&h);
        }
      }
      uint8_t* dst = reinterpret_cast<uint8_t*>(seq_wts + static_cast<size_t>(pg) * kBlock * p.lw);
      uint8_t* lo = dst + (4 * c4) * 16;
      uint8_t* hi = dst + p.lw * 16 + (4 * c4) * 16;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        *reinterpret_cast<uint4*>(lo + j * 16) = make_uint4(w[j][0], w[j][1], w[j][2], w[j][3]);
        *reinterpret_cast<uint4*>(hi + j * 16) = make_uint4(w[j][4], w[j][5], w[j][6], w[j][7]);
      }
    }
  }
  sL[tid] = make_float4(L[0], L[1], L[2], L[3]);
  __syncthreads();
  if (lane_pg == 0) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < gp; ++j) {
      const float4 x = sL[(j << log2tpp) + c4];
      s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
    }
    *reinterpret_cast<float4*>(p.lwpart + (static_cast<size_t>(v) * p.n_pc + pc) * p.Hv + hcol) = s;
  }
}

// ======================================================================= vpass
// Z^T (R-range rows x heads) += C_V^T (R-range x 16 tokens) . P^T (16 x heads)
// per page, with A = the V page slice as an MN-major 128B-swizzled operand
// (exactly the layout TMA writes for 64-element x 16-token boxes) and B = the
// fp16 attention weights in a K-major, unswizzled layout written by the
// P warps (chunked prefill: by chunk_weights_kernel).  The accumulator lives in
// tensor memory: one 128-lane x npad-column block per 128 rows of the R range.
// A ring stage holds up to pps consecutive pages of one segment, so that the
// per-stage work of the single issuing threads (barrier waits, bookkeeping)
// is shared by several pages' copies and MMAs.
struct VPassParams {
  const int32_t* tables;
  const int32_t* row_seq;   // [B] sequence of each row, or null
  const int32_t* teff;
  const int32_t* prefix;
  const float* logits;    // [B][t_pad][H]
  const float* mpart;     // [B][H]: each sequence's max of the logits (decode)
  float* zpart;           // [n_rr][H][v_slots][r_range]: sum_t w c_V per segment
  float* lpart;           // [v_slots][H]: sum_t w per segment (written by R range 0)
  int32_t* status;
  int B, H, npad, MB, NB, R, t_pad, r_range, n_rr, v_slots, stages;
  int n_chunks;           // 64-wide chunks per R range (r_range_pad/64); the last range may hold fewer
  int n_mtiles;           // r_range_pad / 128
  uint32_t tmem_cols;
  uint32_t vtile_bytes;   // r_range_pad*16*2
  uint32_t ltile_bytes;   // 16*H*4
  uint32_t ptile_bytes;   // npad*16*2
  // read-once chunked prefill (vpass_kernel<true>): B counts virtual sequences,
  // logits are [B][n_vg][t_pad][256], the columns are virtual heads h * nq + i
  // (Hv of them, 256 per group: grid y = R range + n_rr * group), and the
  // partials of virtual head (h, i) sit at row (slot * nq + i) of head h
  int Hv, n_vg, log2nq;
  int lw;                 // chunk mode: logits row width = virtual heads per group (npad)
  int pps;                // pages per ring stage (1..kMaxPPS)
  const __half* wts;      // chunk mode: [B][n_vg][t_pad][lw] fp16 weights, each page's tile in the B layout
};
constexpr int kMaxPPS = 8;

constexpr int kVThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 weights + epilogue
constexpr int32_t kFirst = 1, kLast = 2;

// 4 x 4 transpose across a quad of lanes (i = lane & 3): on entry a lane holds
// row i, columns 0..3 of its quad's block; on return rows 0..3 of column i.
// Pairs of lanes first swap the off-diagonal elements of their 2 x 2 blocks,
// then lanes two apart swap the off-diagonal 2 x 2 blocks.
__device__ __forceinline__ float4 quad_transpose(float a0, float a1, float a2, float a3, int i) {
  const bool odd = (i & 1) != 0, upper = (i & 2) != 0;
  const float y0 = __shfl_xor_sync(0xffffffffu, odd ? a0 : a1, 1);
  const float y1 = __shfl_xor_sync(0xffffffffu, odd ? a2 : a3, 1);
  const float b0 = odd ? y0 : a0, b1 = odd ? a1 : y0, b2 = odd ? y1 : a2, b3 = odd ? a3 : y1;
  const float z0 = __shfl_xor_sync(0xffffffffu, upper ? b0 : b2, 2);
  const float z1 = __shfl_xor_sync(0xffffffffu, upper ? b1 : b3, 2);
  return upper ? make_float4(z0, z1, b2, b3) : make_float4(b0, b1, z0, z1);
}

template <bool kChunk>
__global__ void __launch_bounds__(kVThreads, 1)
vpass_kernel(const __grid_constant__ CUtensorMap vmap, VPassParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int S = p.stages, PPS = p.pps;
  const uint32_t vstage = PPS * p.vtile_bytes, lstage = PPS * p.ltile_bytes, pstage = PPS * p.ptile_bytes;
  uint8_t* vtiles = smem;                                               // S x vstage (1024-aligned)
  uint8_t* ltiles = vtiles + static_cast<size_t>(S) * vstage;           // S x lstage
  uint8_t* ptiles = ltiles + static_cast<size_t>(S) * lstage;           // S x pstage
  StageMeta* meta = reinterpret_cast<StageMeta*>(ptiles + static_cast<size_t>(S) * pstage);
  uint64_t* full = reinterpret_cast<uint64_t*>(meta + S);
  uint64_t* pready = full + S;
  uint64_t* empty = pready + S;
  uint64_t* zdone = empty + S;
  uint64_t* tfree = zdone + 1;
  uint64_t* mdone = tfree + 1;
  uint64_t* pbar = mdone + 1;                                           // the weight warps' sync
  float* sM = reinterpret_cast<float*>(pbar + 1);                       // [npad]
  float* sRed = sM + p.npad;                                            // [128]
  __shared__ uint32_t taddr_s;
  __shared__ volatile int32_t abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  griddep_wait();
  griddep_launch_dependents();
  Partition pt;
  pt.P = p.prefix[p.B];
  pt.G = static_cast<int32_t>(pt.P < gridDim.x ? pt.P : gridDim.x);
  const int cta = blockIdx.x;
  const int rr = kChunk ? static_cast<int>(blockIdx.y) % p.n_rr : static_cast<int>(blockIdx.y);
  const int vg = kChunk ? static_cast<int>(blockIdx.y) / p.n_rr : 0;   // group of virtual heads (chunk mode)
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
    mbar_init(pbar, 128);
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
    // The whole warp walks the pages; lane i reads ahead the block-table entry
    // of page cbase + i, so lane 0 issues copies without a dependent global
    // load per page.  Sequence bounds are reloaded only when the walk enters
    // the next sequence.  A stage takes the next min(pps, pages left in the
    // segment) pages: one box per page, one bulk copy for their weights.
    if (lane == 0) prefetch_tensormap(&vmap);
    const uint64_t pol_codes = policy_evict_first();
    const uint64_t pol_logits = policy_evict_first();
    uint32_t k = 0;             // stages issued
    int s = 0;                  // ring slot of stage k
    uint32_t ph = 0;            // parity of that slot's current use
    bool ok = true;
    int32_t b = seq_of_page(p.prefix, p.B, p0);
    int32_t sbeg = p.prefix[b], send = p.prefix[b + 1], T = p.teff[b];
    int64_t cbase = -64;
    int32_t cphys = 0;
    const int c_base = rr * (p.r_range / 64);
    for (int64_t pg_g = p0; pg_g < p1;) {
      while (send <= pg_g) { ++b; sbeg = send; send = p.prefix[b + 1]; T = p.teff[b]; }
      const int32_t pg = static_cast<int32_t>(pg_g - sbeg);
      const int64_t left = (send < p1 ? static_cast<int64_t>(send) : p1) - pg_g;   // pages left in the segment
      const int np = left < PPS ? static_cast<int>(left) : PPS;
      if (pg_g + np > cbase + 32) {
        cbase = pg_g;
        const int64_t xi = pg_g + lane;
        int32_t bi = b;
        while (bi < p.B - 1 && p.prefix[bi + 1] <= xi) ++bi;
        cphys = xi < p1 ? table_row(p.tables, p.row_seq, bi, p.MB)[static_cast<int32_t>(xi - p.prefix[bi])] : 0;
      }
      const int w0 = static_cast<int>(pg_g - cbase);
      int32_t phys[kMaxPPS];
#pragma unroll
      for (int j = 0; j < kMaxPPS; ++j) phys[j] = __shfl_sync(0xffffffffu, cphys, (w0 + j) & 31);
      if (lane == 0) {
        if (k >= static_cast<uint32_t>(S) && !mbar_wait(&empty[s], ph ^ 1u)) {
          ok = false;
        } else {
          int32_t fl = 0;
          if (pg_g == p0 || pg == 0) fl |= kFirst;
          if (np == left) fl |= kLast;   // the stage ends the segment
          const int32_t t0 = pg * kBlock;
          meta[s] = StageMeta{b, t0, min(np * kBlock, T - t0), fl};
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(np) * (static_cast<uint32_t>(p.n_chunks) * 2048u +
                                                                       (kChunk ? p.ptile_bytes : p.ltile_bytes)));
          uint8_t* vt = vtiles + static_cast<size_t>(s) * vstage;
#pragma unroll
          for (int j = 0; j < kMaxPPS; ++j) {
            if (j < np) {
              int32_t pj = phys[j];
              if (pj < 0 || pj >= p.NB) { set_flag(p.status, STARKV_FLAG_BAD_BLOCK_ID); pj = 0; }
              // the page's R range in one box of n_chunks 64-code blocks
              tma_load_3d(vt + j * p.vtile_bytes, &vmap, 0, pj * kBlock, c_base, &full[s], pol_codes);
            }
          }
          if constexpr (kChunk) {
            // the pages' weights, already in the B-operand layout (chunk_weights_kernel)
            const __half* wsrc = p.wts + ((static_cast<size_t>(b) * p.n_vg + vg) * p.t_pad + t0) * p.lw;
            bulk_g2s(ptiles + static_cast<size_t>(s) * pstage, wsrc, np * p.ptile_bytes, &full[s], pol_logits);
          } else {
            bulk_g2s(ltiles + static_cast<size_t>(s) * lstage, p.logits + (static_cast<size_t>(b) * p.t_pad + t0) * p.H,
                     np * p.ltile_bytes, &full[s], pol_logits);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      pg_g += np;
      ++k;
      if (++s == S) { s = 0; ph ^= 1u; }
    }
    if (lane == 0) {
      if (ok) {
        if (k >= static_cast<uint32_t>(S) && !mbar_wait(&empty[s], ph ^ 1u)) ok = false;
        if (ok) { meta[s] = StageMeta{-1, 0, 0, 0}; mbar_arrive(&full[s]); }
      }
      if (!ok) {
        set_timeout(p.status, kSiteVEmpty);
        abort_flag = 1;
      }
      // copies still in flight land before the CTA can exit: the last uses of
      // the ring slots (stage k - S's slot was reused by the end marker)
      const uint32_t first = k >= static_cast<uint32_t>(S) ? k - S + (ok ? 1u : 0u) : 0u;
      for (uint32_t kk = first; kk < k; ++kk) mbar_wait(&full[kk % S], (kk / S) & 1);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, p.npad, /*a_mn_major=*/true, /*b_mn_major=*/false);
      const uint32_t lbo_b = static_cast<uint32_t>(p.npad / 8) * 128u;
      // descriptors of ring slot 0's first page; the start address field
      // (address / 16, 14 bits) advances by plain addition: shared memory
      // addresses stay below 256 KB, so the sum never carries out of it
      const uint64_t adesc0 = smem_desc(smem_u32(vtiles), 2048u, 1024u, kSwizzle128B);
      const uint64_t bdesc0 = smem_desc(smem_u32(ptiles), lbo_b, 128u, kSwizzleNone);
      uint32_t seg = 0;
      uint32_t accumulate = 0;
      int s = 0;
      uint32_t ph = 0;
      for (;;) {
        if (!mbar_wait(&pready[s], ph) || abort_flag) { set_timeout(p.status, kSiteVPready); break; }
        const StageMeta mt = meta[s];
        if (mt.b < 0) break;
        if (mt.flags & kFirst) {
          if (seg > 0 && !mbar_wait(tfree, (seg - 1) & 1)) { set_timeout(p.status, kSiteVTfree); break; }
          accumulate = 0;
        }
        tc_fence_after();
        const int np = (mt.nt + kBlock - 1) >> 4;
        const uint64_t as = adesc0 + ((static_cast<uint32_t>(s) * vstage) >> 4);
        const uint64_t bs = bdesc0 + ((static_cast<uint32_t>(s) * pstage) >> 4);
        for (int j = 0; j < np; ++j) {
          const uint64_t bj = bs + ((static_cast<uint32_t>(j) * p.ptile_bytes) >> 4);
          const uint64_t aj = as + ((static_cast<uint32_t>(j) * p.vtile_bytes) >> 4);
          for (int m = 0; m < p.n_mtiles; ++m)
            umma_f16_ss(taddr + static_cast<uint32_t>(m * p.npad), aj + static_cast<uint32_t>(m * 256), bj, idesc,
                        accumulate);
          accumulate = 1;
        }
        umma_commit(&empty[s]);
        if (mt.flags & kLast) { umma_commit(zdone); ++seg; }
        if (++s == S) { s = 0; ph ^= 1u; }
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
    uint32_t seg = 0, pphase = 0;
    const uint64_t keep = policy_evict_last();   // Z partials: read back by the finish kernel
    int s_next = 0;
    uint32_t ph_next = 0;
    for (;;) {
      const int s = s_next;
      const uint32_t ph = ph_next;
      if (++s_next == S) { s_next = 0; ph_next ^= 1u; }
      // warp-uniform decisions: the TMEM loads of the epilogue are .sync.aligned
      const bool landed = mbar_wait(&full[s], ph);
      if (!__all_sync(0xffffffffu, landed && !abort_flag)) {
        set_timeout(p.status, kSiteVFull);
        abort_flag = 1;
        break;
      }
      const StageMeta mt = meta[s];
      if (mt.b < 0) { mbar_arrive(&pready[s]); break; }
      if (!kChunk && (mt.flags & kFirst)) {   // (chunk mode: the weights arrive with the stage)
        // everyone is done with the previous segment's max
        if (!group_sync(pbar, pphase)) { set_timeout(p.status, kSiteVFull); abort_flag = 1; break; }
        // max of the sequence's logits (merged by the K pass)
        for (int h = et; h < p.npad; h += 128) sM[h] = h < p.H ? p.mpart[static_cast<size_t>(mt.b) * p.H + h] : 0.f;
        if (!group_sync(pbar, pphase)) { set_timeout(p.status, kSiteVFull); abort_flag = 1; break; }
        lsum = 0.f;
      }
      const int np = (mt.nt + kBlock - 1) >> 4;
      const int ntl = mt.nt - ((np - 1) << 4);   // valid tokens of the stage's last page
      if constexpr (!kChunk) {
        const float m_h = sM[h_w];
        for (int j = 0; j < np; ++j) {
          const float* lt = reinterpret_cast<const float*>(ltiles + static_cast<size_t>(s) * lstage +
                                                           static_cast<size_t>(j) * p.ltile_bytes);
          uint8_t* pt_j = ptiles + static_cast<size_t>(s) * pstage + static_cast<size_t>(j) * p.ptile_bytes;
          const int ntj = j == np - 1 ? ntl : kBlock;
          for (int t = t_w0; t < kBlock; t += t_step) {
            // unnormalised weight exp2(s - M) <= 1 (hardware ex2: about 2^-22
            // relative error, far below the fp16 rounding that follows), rounded
            // to fp16 for the MMA; the normaliser sums exactly the rounded weights
            __half w = __float2half_rn(0.f);
            if (t < ntj && h_w < p.H) w = __float2half_rn(ex2_approx(lt[t * p.H + h_w] - m_h));
            lsum += __half2float(w);
            const uint32_t off = static_cast<uint32_t>(t >> 3) * lbo_b + static_cast<uint32_t>(h_w >> 3) * 128u +
                                 static_cast<uint32_t>(h_w & 7) * 16u + static_cast<uint32_t>(t & 7) * 2u;
            *reinterpret_cast<__half*>(pt_j + off) = w;
          }
        }
      }
      if (ntl < kBlock) {
        // tokens past the sequence end: zero their rows of the last page's V
        // tile so that whatever the unused slots hold (NaN included)
        // contributes exactly 0
        uint8_t* vt = vtiles + static_cast<size_t>(s) * vstage + static_cast<size_t>(np - 1) * p.vtile_bytes;
        const int nrows = kBlock - ntl;
        const int n_ch = min(p.n_chunks, (p.R - rr * p.r_range + 63) / 64);
        const int nst = n_ch * nrows * 8;  // 16-byte stores
        for (int x = et; x < nst; x += 128) {
          const int c = x / (nrows * 8), rem = x % (nrows * 8);
          const int t = ntl + rem / 8, u = rem % 8;
          *reinterpret_cast<uint4*>(vt + c * 2048 + t * 128 + u * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&pready[s]);
      if (mt.flags & kLast) {
        const bool done = mbar_wait(zdone, seg & 1);
        if (!__all_sync(0xffffffffu, done)) {
          set_timeout(p.status, kSiteVZdone);
          abort_flag = 1;
          break;
        }
        tc_fence_after();
        const size_t slot = static_cast<size_t>(mt.b) + cta;
        // partial rows [R range][head][slot][r_range]: head h0+hh's row of this slot
        float* zb = p.zpart + ((static_cast<size_t>(rr) * p.H) * p.v_slots + slot) * p.r_range;
        // A block of 32 TMEM columns is stored after a quad transpose
        // (quad_transpose): lane 4g + i then holds column 4k + i of the block
        // at rows 4g .. 4g + 3 of the warp's 32 rows of R, one 16-byte store,
        // and a warp instruction writes 128 contiguous bytes of each of four
        // columns' partial rows.  r_range and R are multiples of 64, so a
        // warp's 32 rows are all inside the R range or all outside it.
        const int i4 = lane & 3;
        if constexpr (kChunk) {
          // virtual head (h, i): row slot * nq + i of head h (npad = lw, a multiple of 32)
          const uint32_t nqm = (1u << p.log2nq) - 1u;
          for (int m = 0; m < p.n_mtiles; ++m) {
            const uint32_t ta = taddr + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(m * p.npad);
            const int j0 = m * 128 + q * 32;   // the warp's first row of the R range
            const bool jok = j0 < p.r_range && rr * p.r_range + j0 < p.R;
            float* zq = p.zpart + j0 + 4 * (lane >> 2);
            for (int h0 = 0; h0 < p.npad; h0 += 32) {
              uint32_t v[32];
              tmem_ld_32x32b_x32(ta + h0, v);
              tmem_ld_wait();
              if (jok) {
                const uint32_t c0 = static_cast<uint32_t>(vg * p.lw + h0);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  const float4 f = quad_transpose(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                                  __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]), i4);
                  const uint32_t col = c0 + 4 * k + i4;
                  const size_t row =
                      ((static_cast<size_t>(rr * p.H + static_cast<int>(col >> p.log2nq)) * p.v_slots + slot)
                       << p.log2nq) + (col & nqm);
                  st_global_hint_free(reinterpret_cast<float4*>(zq + row * p.r_range), f, keep);
                }
              }
            }
          }
        } else {
          // blocks of TMEM columns (M tile m, heads h0 .. h0 + 31), two loaded
          // per wait
          const int nh = (p.H + 31) >> 5;
          const int nblk = p.n_mtiles * nh;
          const size_t hstride = static_cast<size_t>(p.v_slots) * p.r_range;
          auto load_blk = [&](int blk, uint32_t (&v)[32]) {
            const int m = blk / nh, h0 = (blk - m * nh) << 5;
            const uint32_t ta = taddr + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(m * p.npad + h0);
            if (p.npad - h0 >= 32) tmem_ld_32x32b_x32(ta, v);
            else tmem_ld_32x32b_x16(ta, v);
          };
          auto store_blk = [&](int blk, const uint32_t (&v)[32]) {
            const int m = blk / nh, h0 = (blk - m * nh) << 5;
            const int j0 = m * 128 + q * 32;   // the warp's first row of the R range
            if (j0 >= p.r_range || rr * p.r_range + j0 >= p.R) return;   // warp-uniform
            const int kmax = p.npad - h0 >= 32 ? 8 : 4;   // quads of columns loaded
            float* zq = zb + static_cast<size_t>(h0) * hstride + j0 + 4 * (lane >> 2);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              if (k < kmax) {
                const float4 f = quad_transpose(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                                __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]), i4);
                const int hh = 4 * k + i4;
                if (h0 + hh < p.H) st_global_hint_free(reinterpret_cast<float4*>(zq + hh * hstride), f, keep);
              }
            }
          };
          for (int blk = 0; blk < nblk; blk += 2) {
            uint32_t va[32], vb[32];
            load_blk(blk, va);
            if (blk + 1 < nblk) load_blk(blk + 1, vb);
            tmem_ld_wait();
            store_blk(blk, va);
            if (blk + 1 < nblk) store_blk(blk + 1, vb);
          }
        }
        tc_fence_before();
        mbar_arrive(tfree);
        if constexpr (kChunk) {   // the normalisers were summed once by chunk_weights_kernel
          ++seg;
          continue;
        }
        // per-segment normaliser of every head
        sRed[et] = lsum;
        if (!group_sync(pbar, pphase)) { set_timeout(p.status, kSiteVFull); abort_flag = 1; break; }
        if (rr == 0 && et < p.H) {
          float Ls = 0.f;
          for (int i = et; i < 128; i += p.npad) Ls += sRed[i];
          p.lpart[slot * p.H + et] = Ls;
        }
        if (!group_sync(pbar, pphase)) { set_timeout(p.status, kSiteVFull); abort_flag = 1; break; }
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

// ==================================================================== finish
// out_h^T (d x B) = B_V^h^T (d x R) . (Z_h / L)^T (R x B) on tcgen05 tensor
// cores, with Z / L formed on the fly from the V pass's per-segment partials
// (the split reduction of Z and the up-projection in one kernel).
//
// Partials are laid out [R range][head][slot][r_range] (fp32), so for one
// head and one R range the slots of consecutive sequences are consecutive
// rows: sequence b owns slots b + i0 .. b + i1 (the V-pass CTAs i0..i1 that
// overlapped it), and those runs are ordered and disjoint.  A batch tile of
// sequences therefore needs one contiguous block of partial rows, brought in
// per stage (64 rows of R) by 2-D TMA boxes of 32 partial rows x 64 values.
// Four converter warps sum each sequence's rows in segment order, scale by
// 1/L (L = the summed fp16 weights of all its segments) and split the result
// into fp16 hi + lo halves (about 22 bits of the fp32 value), written straight
// into the MMA's B operand (K-major, 128-byte swizzle).  Z / L is a convex
// combination of fp16 codes, so both halves are in range.  A = B_V^h^T from
// 64x64 TMA boxes of B_V (MN-major, 128B swizzle); two MMAs per K step (hi
// and lo).  R is split over a cluster whose partial sums are added through
// distributed shared memory in rank order.
struct FinishParams {
  __half* out;            // [B][H][d]
  const float* zpart;     // the V-pass partials (read directly for tiles too wide to stage)
  const float* lpart;     // [v_slots][H]
  const int32_t* prefix;  // [B+1]
  int B, H, d, R;
  int log2G;              // query head h reads B_V columns of KV head h >> log2G
  int r_range, v_slots, v_grid;
  int n_mt;               // 128-row tiles of d
  int bt_rows;            // sequences per batch tile
  int k_per_cta;          // rows of R per CTA (multiple of 64)
  int npad;               // UMMA N (batch tile padded to 16)
  int stages;
  int zrows;              // partial rows reserved per stage (multiple of kFinZBox, >= any tile's need)
  uint32_t stage_bytes;
  uint32_t tmem_cols;
  // read-once chunked prefill: the "sequences" are virtual sequences of
  // 1 << log2nq query rows; B-operand row v * nq + i is row i of virtual
  // sequence v (output row vs_row0[v] + i, present while i < vs_nrows[v]),
  // its partials are rows slot * nq + i of head h, its normalisers are
  // lpart[slot][h * nq + i] (row width Hv).  log2nq = 0, vs_row0 = null: decode.
  const int32_t* vs_row0;
  const int32_t* vs_nrows;
  int log2nq, Hv;
  const float* lwpart;    // chunk mode: [B][n_pc][Hv] normaliser partials of each virtual head
  int n_pc;
};

constexpr int kFinThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2..9 convert; warps 2..5 drain TMEM
constexpr int kFinConv = kFinThreads - 64;
constexpr int kFinKC = 64;        // rows of R per stage
constexpr int kFinZBox = 32;      // partial rows per TMA box
constexpr int kFinMaxRows = 256;  // sequences per batch tile at most
constexpr int kFinSegBatch = 4;   // partial rows a converter loads before adding them

// First slot (a lower bound) and slot count of the partials of sequences
// [b0, b1) for a V-pass partition pt (P > 0).
__device__ __forceinline__ void tile_slots(const int32_t* prefix, const Partition& pt, int b0, int b1,
                                           int32_t* lo, int32_t* n) {
  const int64_t f0 = min(static_cast<int64_t>(prefix[b0]), pt.P - 1);
  const int64_t f1 = min(max(static_cast<int64_t>(prefix[b1]) - 1, int64_t{0}), pt.P - 1);
  *lo = b0 + part_owner(f0, pt);
  *n = (b1 - 1 + part_owner(f1, pt)) - *lo + 1;
}

// grid (H * n_mt * n_bt, KS), cluster (1, KS, 1)
__global__ void __launch_bounds__(kFinThreads, 1)
finish_kernel(const __grid_constant__ CUtensorMap bvmap, const __grid_constant__ CUtensorMap zmap, FinishParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int S = p.stages;
  const uint32_t a_bytes = 2u * kFinKC * 128u;                      // two 64x64 boxes of B_V
  const uint32_t half_bytes = static_cast<uint32_t>(p.npad) * 128u;  // one hi or lo operand tile
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(S) * p.stage_bytes);
  uint64_t* conv = full + S;
  uint64_t* empty = conv + S;
  uint64_t* done = empty + S;
  int32_t* s_row = reinterpret_cast<int32_t*>(done + 1);            // [kFinMaxRows] first partial row
  int32_t* s_nseg = s_row + kFinMaxRows;                            // [kFinMaxRows] segments
  float* s_il = reinterpret_cast<float*>(s_nseg + kFinMaxRows);     // [kFinMaxRows] 1/L
  float* part = reinterpret_cast<float*>(smem);                     // [npad][128], reuses the ring
  __shared__ uint32_t taddr_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int xi = blockIdx.x;
  const int h = xi % p.H; xi /= p.H;
  const int mt = xi % p.n_mt;
  const int bt = xi / p.n_mt;
  const int ks = blockIdx.y, KS = gridDim.y;
  const int b0 = bt * p.bt_rows;                      // first (virtual) sequence of the tile
  const int nb = min(p.bt_rows, p.B - b0);
  const int nq = 1 << p.log2nq;
  const int k0 = ks * p.k_per_cta;
  const int k1 = min(p.R, k0 + p.k_per_cta);
  const int n_stages = k1 > k0 ? (k1 - k0 + kFinKC - 1) / kFinKC : 0;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&conv[s], kFinConv); mbar_init(&empty[s], 1); }
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

  Partition pt;
  pt.P = p.prefix[p.B];
  pt.G = static_cast<int32_t>(pt.P < p.v_grid ? pt.P : p.v_grid);
  int32_t slot_lo = 0, n_slots = 0;
  if (pt.P > 0) tile_slots(p.prefix, pt, b0, b0 + nb, &slot_lo, &n_slots);
  // the tile's partial rows are staged by TMA when they fit the stage, else
  // the converters read them from global memory (an unusually skewed tile)
  const bool staged = (n_slots << p.log2nq) <= p.zrows;
  const int n_box = (n_slots > 0 && staged) ? ((n_slots << p.log2nq) + kFinZBox - 1) / kFinZBox : 0;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tensormap(&bvmap);
      prefetch_tensormap(&zmap);
      const uint64_t pol = policy_evict_first();
      const int col = (h >> p.log2G) * p.d + mt * 128;
      for (int i = 0; i < n_stages; ++i) {
        const int s = i % S;
        if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1)) { ok = false; break; }
        uint8_t* st = smem + static_cast<size_t>(s) * p.stage_bytes;
        const int kr = k0 + i * kFinKC;
        const int rr = kr / p.r_range, jj = kr - rr * p.r_range;
        mbar_arrive_expect_tx(&full[s], a_bytes + static_cast<uint32_t>(n_box) * kFinZBox * 256u);
        tma_load_2d(st, &bvmap, col, kr, &full[s], pol);
        tma_load_2d(st + kFinKC * 128, &bvmap, col + 64, kr, &full[s], pol);
        const int zrow = ((rr * p.H + h) * p.v_slots + slot_lo) << p.log2nq;
        uint8_t* zdst = st + a_bytes + 2u * half_bytes;
        for (int z = 0; z < n_box; ++z)
          tma_load_2d(zdst + static_cast<size_t>(z) * kFinZBox * 256, &zmap, jj, zrow + z * kFinZBox, &full[s], pol);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------------- MMA
      const uint32_t idesc = idesc_f16_f32(128, p.npad, /*a_mn_major=*/true, /*b_mn_major=*/false);
      for (int i = 0; i < n_stages; ++i) {
        const int s = i % S;
        if (!mbar_wait(&conv[s], (i / S) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + static_cast<size_t>(s) * p.stage_bytes);
        const uint32_t shi = sa + a_bytes, slo = shi + half_bytes;
#pragma unroll
        for (int kk = 0; kk < kFinKC / 16; ++kk) {
          const uint64_t adesc = smem_desc(sa + kk * 16u * 128u, kFinKC * 128u, 1024u, kSwizzle128B);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          umma_f16_ss(taddr, adesc, smem_desc(shi + kk * 32u, 16u, 1024u, kSwizzle128B), idesc, acc);
          umma_f16_ss(taddr, adesc, smem_desc(slo + kk * 32u, 16u, 1024u, kSwizzle128B), idesc, 1u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(done);
    }
  } else {
    // ------------------------------------------------------------ converters
    const int et = tid - 64;                 // 0 .. kFinConv-1
    // each sequence's partial rows (relative to the tile's first slot) and 1/L;
    // L sums the per-segment normalisers in segment order
    for (int bl = et; bl < p.npad; bl += kFinConv) {
      int32_t row = 0, nseg = 0;
      float il = 0.f;
      const int vb = bl >> p.log2nq, qi = bl & (nq - 1);   // (virtual) sequence of the tile, its row
      if (vb < nb && pt.P > 0 && (!p.vs_nrows || qi < p.vs_nrows[b0 + vb])) {
        const int b = b0 + vb;
        const int32_t f0 = p.prefix[b], f1 = p.prefix[b + 1];
        if (f1 > f0) {
          const int32_t i0 = part_owner(f0, pt), i1 = part_owner(f1 - 1, pt);
          float Ls = 0.f;
          if (p.lwpart) {
            const float* lp = p.lwpart + static_cast<size_t>(b) * p.n_pc * p.Hv + (h << p.log2nq) + qi;
            for (int j = 0; j < p.n_pc; ++j) Ls += lp[static_cast<size_t>(j) * p.Hv];
          } else {
            for (int32_t i = i0; i <= i1; i += 4) {   // four loads issued before they are added in order
              float l4[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) l4[u] = i + u <= i1 ? p.lpart[static_cast<size_t>(b + i + u) * p.H + h] : 0.f;
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if (i + u <= i1) Ls += l4[u];
            }
          }
          il = 1.f / Ls;
          row = ((b + i0 - slot_lo) << p.log2nq) + qi;
          nseg = i1 - i0 + 1;
          if (row < 0 || (staged && row + ((nseg - 1) << p.log2nq) >= n_box * kFinZBox)) nseg = 0;   // cannot happen
        }
      }
      s_row[bl] = row;
      s_nseg[bl] = nseg;
      s_il[bl] = il;
    }
    named_bar_sync(1, kFinConv);
    for (int i = 0; i < n_stages; ++i) {
      const int s = i % S;
      const bool landed = mbar_wait(&full[s], (i / S) & 1);
      if (!__all_sync(0xffffffffu, landed)) { ok = false; break; }
      uint8_t* st = smem + static_cast<size_t>(s) * p.stage_bytes;
      uint8_t* hi_t = st + a_bytes;
      const uint8_t* zt = st + a_bytes + 2u * half_bytes;
      // partial rows of this stage: staged rows of 64 values, or global rows of r_range values
      const int kr = k0 + i * kFinKC;
      const int rr = kr / p.r_range;
      const float* zg = p.zpart + ((static_cast<size_t>((rr * p.H + h) * p.v_slots + slot_lo) << p.log2nq) * p.r_range) +
                        (kr - rr * p.r_range);
      const int zstride = staged ? 64 : p.r_range;
      // item = (sequence row bl of the tile, 8-value chunk c of the stage's 64 rows of R)
      for (int item = et; item < p.npad * 8; item += kFinConv) {
        const int bl = item >> 3, c = item & 7;
        float z[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) z[u] = 0.f;
        const int nseg = s_nseg[bl];
        if (nseg > 0) {
          const float* src = (staged ? reinterpret_cast<const float*>(zt) : zg) +
                             static_cast<size_t>(s_row[bl]) * zstride + c * 8;
          const size_t gstep = static_cast<size_t>(nq) * zstride;   // segment g: nq partial rows further on
          // the eight threads of a quarter warp read one row's eight 32-byte
          // items; items c >= 4 take their upper 16 bytes first, so that each
          // load touches eight distinct bank groups.  Segments are loaded four
          // at a time and then added in segment order.
          const int h0 = c >> 2;
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f), e = a;
          for (int g0 = 0; g0 < nseg; g0 += kFinSegBatch) {
            float4 v0[kFinSegBatch], v1[kFinSegBatch];
#pragma unroll
            for (int u = 0; u < kFinSegBatch; ++u) {
              if (g0 + u < nseg) {
                const float4* s4 = reinterpret_cast<const float4*>(src + (g0 + u) * gstep);
                v0[u] = s4[h0];
                v1[u] = s4[h0 ^ 1];
              }
            }
#pragma unroll
            for (int u = 0; u < kFinSegBatch; ++u) {
              if (g0 + u < nseg) {
                a.x += v0[u].x; a.y += v0[u].y; a.z += v0[u].z; a.w += v0[u].w;
                e.x += v1[u].x; e.y += v1[u].y; e.z += v1[u].z; e.w += v1[u].w;
              }
            }
          }
          const float4 lo4 = h0 ? e : a, hi4 = h0 ? a : e;
          const float il = s_il[bl];
          z[0] = lo4.x * il; z[1] = lo4.y * il; z[2] = lo4.z * il; z[3] = lo4.w * il;
          z[4] = hi4.x * il; z[5] = hi4.y * il; z[6] = hi4.z * il; z[7] = hi4.w * il;
        }
        uint4 hv, lv;
        uint32_t* hw = reinterpret_cast<uint32_t*>(&hv);
        uint32_t* lw = reinterpret_cast<uint32_t*>(&lv);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const __half2 hh = __floats2half2_rn(z[2 * u], z[2 * u + 1]);
          const float2 g = __half22float2(hh);
          const __half2 ll = __floats2half2_rn(z[2 * u] - g.x, z[2 * u + 1] - g.y);
          hw[u] = *reinterpret_cast<const uint32_t*>(&hh);
          lw[u] = *reinterpret_cast<const uint32_t*>(&ll);
        }
        // K-major operand row bl, 16-byte chunk c at its 128B-swizzled position
        const uint32_t off = static_cast<uint32_t>(bl) * 128u + (static_cast<uint32_t>(c ^ (bl & 7)) << 4);
        *reinterpret_cast<uint4*>(hi_t + off) = hv;
        *reinterpret_cast<uint4*>(hi_t + half_bytes + off) = lv;
      }
      fence_proxy_async_smem();
      mbar_arrive(&conv[s]);
    }
  }
  __syncthreads();
  if (!mbar_wait(done, 0)) ok = false;
  tc_fence_after();
  if (warp >= 2 && warp < 6) {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    for (int c0 = 0; c0 < p.npad; c0 += 16) {
      uint32_t v[32];
      tmem_ld_32x32b_x16(taddr + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int jx = 0; jx < 16; ++jx)
        part[(c0 + jx) * 128 + row] = (n_stages > 0 && ok) ? __uint_as_float(v[jx]) : 0.f;
    }
  }
  tc_fence_before();
  cluster.sync();
  // rank ks sums rows [ks*npad/KS, (ks+1)*npad/KS) over the cluster in rank
  // order, four consecutive outputs per thread (all ranks' loads issued first)
  const int per = (p.npad + KS - 1) / KS;
  const int n_lo = ks * per, n_hi = min(p.npad, n_lo + per);
  for (int x = tid; x < (n_hi - n_lo) * 32; x += kFinThreads) {
    const int n = n_lo + x / 32, m = (x % 32) * 4;
    const int dm = mt * 128 + m;
    const int vb = n >> p.log2nq, qi = n & (nq - 1);
    if (vb >= nb || dm >= p.d) continue;
    if (p.vs_nrows && qi >= p.vs_nrows[b0 + vb]) continue;
    const int64_t orow = p.vs_row0 ? static_cast<int64_t>(p.vs_row0[b0 + vb]) + qi : b0 + n;
    float4 v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < KS) v[c] = *reinterpret_cast<const float4*>(cluster.map_shared_rank(part, c) + n * 128 + m);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < KS) { acc.x += v[c].x; acc.y += v[c].y; acc.z += v[c].z; acc.w += v[c].w; }
    const __half2 lo = __floats2half2_rn(acc.x, acc.y), hi = __floats2half2_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p.out + (static_cast<size_t>(orow) * p.H + h) * p.d + dm) = pk;
  }
  cluster.sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(taddr, p.tmem_cols);
  }
}

}  // namespace starkv
