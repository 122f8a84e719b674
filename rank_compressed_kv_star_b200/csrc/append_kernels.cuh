// Compress-and-append: codes of one new token per sequence into the paged pools.
//
// c_K[b,h,:] = k[b,h,:] . A_K[h]  (head-wise K, A_K[h] is d x r)
// c_V[b,:]   = v[b,:] . A_V       (joint V over the concatenated heads, A_V is H*d x R)
// Both are accumulated in fp32, rounded to fp16 (nearest even) and stored in
// slot pos % 16 of page block_table[b][pos / 16] (Proxima README, method
// paragraph: codes "stored in a compressed paged format").
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace starkv {

struct AppendParams {
  const __half* k;         // [B][H][d]
  const __half* v;         // [B][H*d]
  const __half* A_K;       // [H][d][r]
  const __half* A_V;       // [H*d][R]
  const int32_t* tables;   // [B][MB]
  const int32_t* positions;
  __half* k_cache;         // [NB][16][H][r]
  __half* v_cache;         // [NB][16][R]
  int B, H, d, r, R, MB, NB;
  int nvx, nby;            // V column tiles (64 wide) and batch tiles (16)
};

constexpr int kAppBT = 16;   // sequences per V tile
constexpr int kAppNC = 64;   // code columns per V tile
constexpr int kAppJC = 256;  // input rows staged per pass

// Physical row (page*16 + slot) of sequence b's append target, or -1.
__device__ __forceinline__ int64_t append_row(const AppendParams& p, int b) {
  const int32_t pos = p.positions[b];
  if (pos < 0 || pos / 16 >= p.MB) return -1;
  const int32_t phys = p.tables[static_cast<size_t>(b) * p.MB + pos / 16];
  if (phys < 0 || phys >= p.NB) return -1;
  return static_cast<int64_t>(phys) * 16 + (pos % 16);
}

// grid: nvx*nby V tiles followed by H K blocks; 256 threads.
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nv_blocks = p.nvx * p.nby;
  if (static_cast<int>(blockIdx.x) < nv_blocks) {
    // ---- V: 64 code columns x 16 sequences; 8 warps split the H*d rows of each pass
    __shared__ __align__(16) __half vs[kAppJC][kAppBT];
    __shared__ float red[8][kAppNC][kAppBT + 1];
    const int nx = blockIdx.x % p.nvx, by = blockIdx.x / p.nvx;
    const int n0 = nx * kAppNC, b0 = by * kAppBT;
    const int HD = p.H * p.d;
    float acc[kAppBT][2];
#pragma unroll
    for (int u = 0; u < kAppBT; ++u) acc[u][0] = acc[u][1] = 0.f;
    for (int jc = 0; jc < HD; jc += kAppJC) {
      __syncthreads();
      for (int x = tid; x < kAppJC * kAppBT; x += 256) {
        const int bb = x / kAppJC, jj = x % kAppJC;
        const int b = b0 + bb, j = jc + jj;
        vs[jj][bb] = (b < p.B && j < HD) ? p.v[static_cast<size_t>(b) * HD + j] : __float2half_rn(0.f);
      }
      __syncthreads();
      const int jn = min(kAppJC, HD - jc);
      for (int jj = warp * (kAppJC / 8); jj < (warp + 1) * (kAppJC / 8) && jj < jn; ++jj) {
        const float2 a = __half22float2(
            *reinterpret_cast<const __half2*>(p.A_V + static_cast<size_t>(jc + jj) * p.R + n0 + 2 * lane));
        const uint4* vr = reinterpret_cast<const uint4*>(&vs[jj][0]);
        const uint4 w0 = vr[0], w1 = vr[1];
        const __half2* h0 = reinterpret_cast<const __half2*>(&w0);
        const __half2* h1 = reinterpret_cast<const __half2*>(&w1);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 x0 = __half22float2(h0[u]);
          const float2 x1 = __half22float2(h1[u]);
          acc[2 * u][0] = fmaf(x0.x, a.x, acc[2 * u][0]);
          acc[2 * u][1] = fmaf(x0.x, a.y, acc[2 * u][1]);
          acc[2 * u + 1][0] = fmaf(x0.y, a.x, acc[2 * u + 1][0]);
          acc[2 * u + 1][1] = fmaf(x0.y, a.y, acc[2 * u + 1][1]);
          acc[8 + 2 * u][0] = fmaf(x1.x, a.x, acc[8 + 2 * u][0]);
          acc[8 + 2 * u][1] = fmaf(x1.x, a.y, acc[8 + 2 * u][1]);
          acc[8 + 2 * u + 1][0] = fmaf(x1.y, a.x, acc[8 + 2 * u + 1][0]);
          acc[8 + 2 * u + 1][1] = fmaf(x1.y, a.y, acc[8 + 2 * u + 1][1]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kAppBT; ++u) {
      red[warp][2 * lane][u] = acc[u][0];
      red[warp][2 * lane + 1][u] = acc[u][1];
    }
    __syncthreads();
    for (int x = tid; x < kAppNC * kAppBT; x += 256) {
      const int c = x % kAppNC, bb = x / kAppNC;
      const int b = b0 + bb;
      if (b >= p.B) continue;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) s += red[w][c][bb];
      const int64_t row = append_row(p, b);
      if (row >= 0) p.v_cache[row * p.R + n0 + c] = __float2half_rn(s);
    }
    return;
  }
  // ---- K: one block per head; thread = (rank index, sequence lane)
  const int h = blockIdx.x - nv_blocks;
  const int i = tid % p.r;
  const int bpar = 256 / p.r;
  const int bs = tid / p.r;
  if (bs >= bpar) return;
  const __half* A = p.A_K + static_cast<size_t>(h) * p.d * p.r + i;
  for (int b = bs; b < p.B; b += bpar) {
    const __half* krow = p.k + (static_cast<size_t>(b) * p.H + h) * p.d;
    float acc = 0.f;
    for (int j = 0; j < p.d; ++j) acc = fmaf(__half2float(krow[j]), __half2float(A[static_cast<size_t>(j) * p.r]), acc);
    const int64_t row = append_row(p, b);
    if (row >= 0) p.k_cache[(row * p.H + h) * p.r + i] = __float2half_rn(acc);
  }
}

}  // namespace starkv
