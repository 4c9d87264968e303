// elementwise.cuh — the two memory-bound helpers of the path:
//   k_fold     weight folding, W*[n][k] = RNE_bf16(g[k] * W[k][n]) written K-major (transposed), with
//              the GLU gate/up block interleave ("FlashNorm: Fast Normalization for Transformers",
//              Abstract, item i: folding the normalization weights into the next linear layer).
//   k_rmsnorm  the first kernel of the unfused baseline: xn = RNE_bf16(x / sqrt(mean(x^2)+eps) * g).
#pragma once

#include "sm100.cuh"

namespace fn {

constexpr int kFoldTile = 64;

// Destination row of source column `c` of W. Linear: identity. GLU (N = 2F): gate column j goes to
// row 32*(j/16) + j%16, up column F + j to row 32*(j/16) + 16 + j%16.
__device__ __forceinline__ int fold_dst_row(int c, int F, bool glu) {
  if (!glu) return c;
  const bool up = c >= F;
  const int j = up ? c - F : c;
  return ((j >> 4) << 5) + (up ? 16 : 0) + (j & 15);
}

// One 64 x 64 tile of W per block (256 threads): coalesced 16-byte loads along n, a transpose in
// shared memory, coalesced 16-byte stores along k. d % 8 == 0 and N % 8 == 0.
__global__ void __launch_bounds__(256) k_fold(const uint16_t* __restrict__ W, const uint16_t* __restrict__ g,
                                              uint16_t* __restrict__ Wstar, int d, int N, int glu) {
  __shared__ uint16_t tile[kFoldTile][kFoldTile + 2];  // [n][k]
  const int k0 = blockIdx.y * kFoldTile;
  const int n0 = blockIdx.x * kFoldTile;
  const int F = N / 2;
  grid_dep_wait();
  // load: 64 rows (k) x 8 chunks of 8 columns (n)
  for (int i = threadIdx.x; i < kFoldTile * 8; i += 256) {
    const int kk = i >> 3, ch = i & 7;
    const int k = k0 + kk, n = n0 + ch * 8;
    if (k < d && n < N) {
      const uint4 v = *reinterpret_cast<const uint4*>(W + static_cast<size_t>(k) * N + n);
      const float gk = __uint_as_float(static_cast<uint32_t>(g[k]) << 16);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // bf16 x bf16 is exact in fp32; cvt.rn rounds it once to bf16.
        const uint32_t packed = pack_bf16x2(gk * bf16lo_to_f32(w[e]), gk * bf16hi_to_f32(w[e]));
        tile[ch * 8 + 2 * e][kk] = static_cast<uint16_t>(packed & 0xFFFFu);
        tile[ch * 8 + 2 * e + 1][kk] = static_cast<uint16_t>(packed >> 16);
      }
    }
  }
  __syncthreads();
  // store: 64 rows (n) x 8 chunks of 8 k-values
  for (int i = threadIdx.x; i < kFoldTile * 8; i += 256) {
    const int nn = i >> 3, ch = i & 7;
    const int n = n0 + nn, k = k0 + ch * 8;
    if (n < N && k < d) {
      uint4 v;
      uint32_t* pv = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        pv[e] = static_cast<uint32_t>(tile[nn][ch * 8 + 2 * e]) |
                (static_cast<uint32_t>(tile[nn][ch * 8 + 2 * e + 1]) << 16);
      const int r = fold_dst_row(n, F, glu != 0);
      *reinterpret_cast<uint4*>(Wstar + static_cast<size_t>(r) * d + k) = v;
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp per row, 8 rows per block. Pass 1 sums squares, pass 2 (L1/L2 hits) scales and stores.
// LayerNorm fold, part 2: colsum[n] = sum_k W*[n][k] over the bf16 values of the folded weight (the
// operand the MMA multiplies), one warp per output column n (a contiguous K-major row of W*).
__global__ void __launch_bounds__(256) k_ln_colsum(const uint16_t* __restrict__ Wstar, float* __restrict__ colsum,
                                                   int d, int N) {
  grid_dep_wait();
  const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (n >= N) return;
  const uint16_t* row = Wstar + static_cast<size_t>(n) * d;
  float s = 0.0f;
  for (int k = lane; k < d; k += 32) s += __uint_as_float(static_cast<uint32_t>(row[k]) << 16);
  s = warp_sum(s);
  if (lane == 0) colsum[n] = s;
}

// LayerNorm fold, part 3: bias[n] = sum_k beta[k] W[k][n] (W row-major [d, N]; beta == nullptr gives 0),
// one thread per column, fp32 products of the exact bf16 values.
__global__ void __launch_bounds__(256) k_ln_bias(const uint16_t* __restrict__ W, const uint16_t* __restrict__ beta,
                                                 float* __restrict__ bias, int d, int N) {
  grid_dep_wait();
  const int n = blockIdx.x * 256 + threadIdx.x;
  if (n >= N) return;
  float s = 0.0f;
  if (beta != nullptr)
    for (int k = 0; k < d; ++k)
      s = fmaf(__uint_as_float(static_cast<uint32_t>(beta[k]) << 16),
               __uint_as_float(static_cast<uint32_t>(W[static_cast<size_t>(k) * N + n]) << 16), s);
  bias[n] = s;
}

// RoPE (cos, sin) table, fp32 [max_pos][head_dim/2][2]: pair i of position p is rotated by the angle
// p * base^(-2i/head_dim) (RoFormer's rotary embedding). The angle and its cosine and sine are taken in
// double precision (the CUDA math library's pow and sincos), then rounded once to fp32.
__global__ void __launch_bounds__(256) k_rope_table(float* __restrict__ cs, int max_pos, int head_dim, double base) {
  grid_dep_wait();
  const int half = head_dim / 2;
  const long long n = static_cast<long long>(max_pos) * half;
  for (long long e = blockIdx.x * 256ll + threadIdx.x; e < n; e += static_cast<long long>(gridDim.x) * 256) {
    const int p = static_cast<int>(e / half), i = static_cast<int>(e % half);
    const double ang = static_cast<double>(p) * pow(base, -2.0 * i / head_dim);
    double s, c;
    sincos(ang, &s, &c);
    reinterpret_cast<float2*>(cs)[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

// Failure-detection self-test: one thread waits on an mbarrier that nothing will ever arrive at. The
// bounded wait runs out after limit_ns (and as many SM cycles), records the timeout in the device
// status word and the kernel returns normally.
__global__ void __launch_bounds__(32) k_wait_selftest(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_init_fence();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait_limited(&bar, 0, &abort_flag, limit_ns, static_cast<long long>(limit_ns));
}

__global__ void __launch_bounds__(256) k_rmsnorm(const uint16_t* __restrict__ x, const uint16_t* __restrict__ g,
                                                 uint16_t* __restrict__ xn, int M, int K, float eps) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  grid_dep_wait();
  if (row >= M) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(row) * K);
  const uint4* gr = reinterpret_cast<const uint4*>(g);
  uint4* outr = reinterpret_cast<uint4*>(xn + static_cast<size_t>(row) * K);
  const int kc = K >> 3;
  float s0 = 0.f, s1 = 0.f;
  for (int c = lane; c < kc; c += 32) {
    const uint4 v = xr[c];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = bf16lo_to_f32(w[e]), b = bf16hi_to_f32(w[e]);
      s0 = fmaf(a, a, s0);
      s1 = fmaf(b, b, s1);
    }
  }
  const float ss = warp_sum(s0 + s1);
  const float r = 1.0f / sqrtf(ss / static_cast<float>(K) + eps);
  for (int c = lane; c < kc; c += 32) {
    const uint4 v = xr[c];
    const uint4 gv = gr[c];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o[e] = pack_bf16x2(bf16lo_to_f32(w[e]) * r * bf16lo_to_f32(gw[e]),
                         bf16hi_to_f32(w[e]) * r * bf16hi_to_f32(gw[e]));
    outr[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace fn
