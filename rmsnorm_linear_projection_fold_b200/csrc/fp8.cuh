// fp8.cuh — quantized W*: the gain fold followed by per-output-channel FP8 E4M3 weight quantization,
// and the decode GEMV that streams the one-byte weights.
//
// The FlashNorm abstract notes that folded checkpoints stay compatible with quantized models: the gain
// is folded into the weight BEFORE quantization, and the deferred 1/rms multiplies the output together
// with the channel's dequantization scale:
//     W*[n, k] = g[k] W[k, n]                  (exact in fp32: bf16 x bf16)
//     s[n]     = max_k |W*[n, k]| / 448          (1 for an all-zero channel)
//     Q[n, k]  = e4m3_rn_satfinite(W*[n, k] / s[n])
//     y[m, n]  = (sum_k x[m, k] Q[n, k]) * s[n] * 1/sqrt(mean_k x[m, k]^2 + eps)
// Decode streams Q (one byte per weight: half the bytes of bf16 W*) with x staged in shared memory, as
// the bf16 GEMV does; each 16-byte load carries 16 weights.
//
// The same abstract item, with NVFP4 (4-bit) weights: E2M1 codes, one E4M3 scale per 16 consecutive k of
// a channel, and a per-channel fp32 scale in place of the format's per-tensor one:
//     s2[n]    = max_k |W*[n, k]| / (448 * 6)   (1 for an all-zero channel)
//     sb[n, b] = e4m3_rn_satfinite(max_{k in b} |W*[n, k]| / (6 * s2[n]))
//     Q[n, k]  = e2m1_rn_satfinite(W*[n, k] / (sb[n, b] * s2[n]))   (0 where sb is 0)
//     y[m, n]  = (sum_k x[m, k] Q[n, k] sb[n, k / 16]) * s2[n] * 1/sqrt(mean_k x[m, k]^2 + eps)
// stored per channel in groups of 256 k of 144 bytes: 32 words of codes (word j: k = 8 j .. 8 j + 7 of the
// group, the even k in bits 0..15, four bits each, the odd k in bits 16..31), then the 16 block scales.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "elementwise.cuh"
#include "gemv.cuh"
#include "sm100.cuh"

namespace fn {

constexpr float kE4m3Max = 448.0f;

// s[n] for every output channel: one thread per column n of W [d, N] (row-major), reads coalesced
// across the threads of a warp.
__global__ void __launch_bounds__(256) k_fp8_scales(const uint16_t* __restrict__ W, const uint16_t* __restrict__ g,
                                                    float* __restrict__ scales, int d, int N, float div) {
  grid_dep_wait();
  const int n = blockIdx.x * 256 + threadIdx.x;
  if (n >= N) return;
  float amax = 0.0f;
  for (int k = 0; k < d; ++k) {
    const float v = __uint_as_float(static_cast<uint32_t>(g[k]) << 16) *
                    __uint_as_float(static_cast<uint32_t>(W[static_cast<size_t>(k) * N + n]) << 16);
    amax = fmaxf(amax, fabsf(v));
  }
  scales[n] = amax > 0.0f ? __fdiv_rn(amax, div) : 1.0f;  // div: 448 (FP8), 448 * 6 (NVFP4)
}

constexpr float kNvfp4ScaleDiv = 448.0f * 6.0f;
constexpr int kNvfp4Group = 256;       // k per stored group
constexpr int kNvfp4GroupBytes = 144;  // 128 bytes of codes + 16 block scales

// E2M1 code of t: round to nearest, ties to even, saturating at +-6. The magnitudes are 0, 0.5, 1, 1.5, 2,
// 3, 4, 6 (codes 0..7); each comparison below is one midpoint between neighbours, strict where the lower
// neighbour has the even code (it takes the tie), inclusive where the upper one has. The sign is kept.
__device__ __forceinline__ uint32_t e2m1_rn_satfinite(float t) {
  const float a = fabsf(t);
  const uint32_t m = static_cast<uint32_t>(a > 0.25f) + static_cast<uint32_t>(a >= 0.75f) +
                     static_cast<uint32_t>(a > 1.25f) + static_cast<uint32_t>(a >= 1.75f) +
                     static_cast<uint32_t>(a > 2.5f) + static_cast<uint32_t>(a >= 3.5f) + static_cast<uint32_t>(a > 5.0f);
  return m | ((__float_as_uint(t) >> 28) & 8u);
}

// One block per (32 channels, one 256-k group): W* of the group through shared memory ([n][k], one thread
// per k on the way in, loads of 8 channels at a time), then one thread per (channel, 16-k block): the
// block's E4M3 scale and its 16 E2M1 codes in the stored layout. Blocks past d get zero codes and a zero
// scale. d % 16 == 0, N % 8 == 0.
__global__ void __launch_bounds__(256) k_fold_nvfp4(const uint16_t* __restrict__ W, const uint16_t* __restrict__ g,
                                                    const float* __restrict__ s2, uint8_t* __restrict__ Q4, int d,
                                                    int N) {
  __shared__ float tile[32][kNvfp4Group + 1];  // [n][k]: +1 keeps the column writes on distinct banks
  const int groups = (d + kNvfp4Group - 1) / kNvfp4Group;
  const int n0 = blockIdx.x * 32, grp = blockIdx.y;
  grid_dep_wait();
  {
    const int kk = threadIdx.x, k = grp * kNvfp4Group + kk;
    const float gk = k < d ? bf16lo_to_f32(g[k]) : 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int n = n0 + 8 * c;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (k < d && n < N) v = *reinterpret_cast<const uint4*>(W + static_cast<size_t>(k) * N + n);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        tile[8 * c + 2 * e][kk] = gk * bf16lo_to_f32(w[e]);  // exact: a bf16 x bf16 product fits fp32
        tile[8 * c + 2 * e + 1][kk] = gk * bf16hi_to_f32(w[e]);
      }
    }
  }
  __syncthreads();
  for (int item = threadIdx.x; item < 32 * 16; item += 256) {
    const int nn = item >> 4, bb = item & 15, n = n0 + nn;
    if (n >= N) continue;
    const float* v = &tile[nn][bb * 16];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
    const float sc2 = s2[n];
    const float t = __fdiv_rn(amax, __fmul_rn(6.0f, sc2));
    const uint32_t sbc = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(t, t), __NV_SATFINITE, __NV_E4M3)) & 0xFFu;
    const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(sbc), __NV_E4M3);
    const float den = __fmul_rn(__half2float(__half(hr)), sc2);  // the decoded scale is exact in half
    uint32_t words[2] = {0u, 0u};
    if (den > 0.0f) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t q = e2m1_rn_satfinite(__fdiv_rn(v[j], den));
        const int jj = j & 7;
        words[j >> 3] |= q << ((jj & 1) * 16 + (jj >> 1) * 4);
      }
    }
    uint8_t* row = Q4 + static_cast<size_t>(n) * groups * kNvfp4GroupBytes + static_cast<size_t>(grp) * kNvfp4GroupBytes;
    *reinterpret_cast<uint2*>(row + bb * 8) = make_uint2(words[0], words[1]);
    row[128 + bb] = static_cast<uint8_t>(sbc);
  }
}

// Q [N, d] (K-major, one byte per weight) from W [d, N], g and the scales: one 64 x 64 tile per block,
// loads along n, a transpose through shared memory, 16-byte stores along k. d % 16 == 0, N % 8 == 0.
__global__ void __launch_bounds__(256) k_fold_fp8(const uint16_t* __restrict__ W, const uint16_t* __restrict__ g,
                                                  const float* __restrict__ scales, uint8_t* __restrict__ Q, int d,
                                                  int N) {
  __shared__ uint8_t tile[kFoldTile][kFoldTile + 16];  // [n][k]
  const int k0 = blockIdx.y * kFoldTile;
  const int n0 = blockIdx.x * kFoldTile;
  grid_dep_wait();
  for (int i = threadIdx.x; i < kFoldTile * 8; i += 256) {
    const int kk = i >> 3, ch = i & 7;
    const int k = k0 + kk, n = n0 + ch * 8;
    if (k < d && n < N) {
      const uint4 v = *reinterpret_cast<const uint4*>(W + static_cast<size_t>(k) * N + n);
      const float gk = __uint_as_float(static_cast<uint32_t>(g[k]) << 16);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int nn = ch * 8 + 2 * e + h;
          const float q = __fdiv_rn(gk * (h ? bf16hi_to_f32(w[e]) : bf16lo_to_f32(w[e])), scales[n0 + nn]);
          // both halves of the pair get the same value, so the byte order of the packed result is moot
          const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(make_float2(q, q), __NV_SATFINITE, __NV_E4M3);
          tile[nn][kk] = static_cast<uint8_t>(c & 0xFFu);
        }
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kFoldTile * 4; i += 256) {
    const int nn = i >> 2, ch = i & 3;
    const int n = n0 + nn, k = k0 + ch * 16;
    if (n < N && k < d) {
      uint4 v;
      uint8_t* pv = reinterpret_cast<uint8_t*>(&v);
#pragma unroll
      for (int e = 0; e < 16; ++e) pv[e] = tile[nn][ch * 16 + e];
      *reinterpret_cast<uint4*>(Q + static_cast<size_t>(n) * d + k) = v;
    }
  }
}

__device__ __forceinline__ uint4 ldg_stream_b(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Four E4M3 codes of one 32-bit word -> fp32, in memory order (E4M3 values are exact in f16 and f32).
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t w, float (&f)[4]) {
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
  f[0] = __half2float(__half(__half_raw{lo.x}));
  f[1] = __half2float(__half(__half_raw{lo.y}));
  f[2] = __half2float(__half(__half_raw{hi.x}));
  f[3] = __half2float(__half(__half_raw{hi.y}));
}

// 16 weights (one 16-byte load) against 16 x values (two 16-byte chunks of bf16).
__device__ __forceinline__ float dot16_fp8(const uint4& q, const uint4& x0, const uint4& x1, float acc) {
  const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
  const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float f[4];
    e4m3x4_to_f32(qw[e], f);
    acc = fmaf(f[0], bf16lo_to_f32(xw[2 * e]), acc);
    acc = fmaf(f[1], bf16hi_to_f32(xw[2 * e]), acc);
    acc = fmaf(f[2], bf16lo_to_f32(xw[2 * e + 1]), acc);
    acc = fmaf(f[3], bf16hi_to_f32(xw[2 * e + 1]), acc);
  }
  return acc;
}

// The FP8 decode GEMV: as k_gemv (linear), with one-byte weights and the channel scale in the epilogue.
// (Measured against two variants on the Llama-7B QKV decode: x widened to fp32 in shared memory with
// packed fp32x2 FMAs, and an integer-only E4M3 decode; both were slower than this hardware-conversion form.)
// MT: rows of x held (>= M, power of two). R: output columns per warp step.
template <int MT, int R, bool OUT_F32>
__global__ void __launch_bounds__(kGemvThreads) k_gemv_fp8(const uint16_t* __restrict__ x,
                                                           const uint8_t* __restrict__ q,
                                                           const float* __restrict__ scales, void* __restrict__ y,
                                                           int M, int K, int N, float eps) {
  extern __shared__ uint4 smem_v[];
  uint4* xs = smem_v;  // [MT][K/8] chunks of 8 bf16
  float* rs = reinterpret_cast<float*>(reinterpret_cast<uint16_t*>(smem_v) + MT * K);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kc = K >> 3;   // x chunks per row
  const int qc = K >> 4;   // 16-weight chunks per W* row
  {
    // this warp's first group of codes into L2 (up to 4 KB a row) while the previous kernel drains
    const int u = (static_cast<int>(blockIdx.x) * (kGemvThreads / 32) + warp) * R + lane;
    if (lane < R && u < N) bulk_prefetch_l2(q + static_cast<size_t>(u) * K, static_cast<uint32_t>(min(K, 4096) & ~15));
  }
  grid_dep_wait();

  for (int i = threadIdx.x; i < MT * kc; i += kGemvThreads) {
    const int m = i / kc, c = i - m * kc;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (m < M) v = *reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * K + c * 8);
    xs[i] = v;
  }
  __syncthreads();
  for (int m = warp; m < MT; m += kGemvThreads / 32) {
    float s0 = 0.f, s1 = 0.f;
    for (int c = lane; c < kc; c += 32) {
      const uint4 v = xs[m * kc + c];
      const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16lo_to_f32(ww[e]), b = bf16hi_to_f32(ww[e]);
        s0 = fmaf(a, a, s0);
        s1 = fmaf(b, b, s1);
      }
    }
    const float ss = warp_sum(s0 + s1);
    if (lane == 0) rs[m] = 1.0f / sqrtf(ss / static_cast<float>(K) + eps);
  }
  __syncthreads();

  const int groups = (N + R - 1) / R;
  for (int gi = blockIdx.x * (kGemvThreads / 32) + warp; gi < groups; gi += gridDim.x * (kGemvThreads / 32)) {
    const uint8_t* rows[R];
    bool valid[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int u = gi * R + i;
      valid[i] = u < N;
      rows[i] = q + static_cast<size_t>(valid[i] ? u : 0) * K;
    }
    float acc[MT][R];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int j = 0; j < R; ++j) acc[m][j] = 0.f;

    for (int c0 = lane; c0 < qc; c0 += 32 * kGemvUnroll) {
      uint4 wv[kGemvUnroll][R];
#pragma unroll
      for (int uu = 0; uu < kGemvUnroll; ++uu) {
        const int c = c0 + uu * 32;
#pragma unroll
        for (int j = 0; j < R; ++j)
          wv[uu][j] = (c < qc && valid[j]) ? ldg_stream_b(rows[j] + c * 16) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int uu = 0; uu < kGemvUnroll; ++uu) {
        const int c = c0 + uu * 32;
        if (c < qc) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const uint4 x0 = xs[m * kc + 2 * c], x1 = xs[m * kc + 2 * c + 1];
#pragma unroll
            for (int j = 0; j < R; ++j) acc[m][j] = dot16_fp8(wv[uu][j], x0, x1, acc[m][j]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int j = 0; j < R; ++j) acc[m][j] = warp_sum(acc[m][j]);

    // lane l writes column (l % R) of row (l / R)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
      for (int i = 0; i < R; ++i) {
        if (lane == ((m * R + i) & 31) && m < M) {
          const int u = gi * R + i;
          if (u < N) {
            const float v = acc[m][i] * scales[u] * rs[m];
            if (OUT_F32)
              static_cast<float*>(y)[static_cast<size_t>(m) * N + u] = v;
            else
              static_cast<uint16_t*>(y)[static_cast<size_t>(m) * N + u] =
                  static_cast<uint16_t>(pack_bf16x2(v, 0.f) & 0xFFFFu);
          }
        }
      }
    }
  }
}

}  // namespace fn
