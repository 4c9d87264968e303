// gemv.cuh — the decode path (M <= 16 tokens): the same deferred FlashNorm computation,
//     y[m, n] = (sum_k x[m,k] W*[n,k]) * 1/sqrt(mean_k x[m,k]^2 + eps)
// as a bandwidth-bound GEMV. In decode the time goes into launching work and moving W* through HBM,
// not into arithmetic (the talk page "Weight Folding, CUDA Streams, and the Bug That Made My Model
// Speak Backwards" makes this point about RMSNorm firing many times per decode step). Folding removes
// the gain tensor from the stream; deferral lets the sum of squares be computed from the x rows
// already staged in shared memory while the W* loads are in flight.
//
// Each block stages x[M, K] (bf16) in shared memory and computes 1/rms per row. Each warp then owns R
// output columns at a time: every lane streams 16-byte chunks of the R rows of W* (K-major, so each
// row is contiguous), multiplies them with the matching x chunks from shared memory for all M rows,
// and the warp reduces with shuffles. GLU units read the gate row and its up row (32*(j/16) + j%16 and
// +16) and apply silu(r*gate) * (r*up).
#pragma once

#include "elementwise.cuh"
#include "sm100.cuh"

namespace fn {

constexpr int kGemvThreads = 256;
constexpr int kGemvUnroll = 4;

__device__ __forceinline__ uint4 ldg_stream(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float dot8(const uint4& a, const uint4& b, float acc) {
  acc = fmaf(bf16lo_to_f32(a.x), bf16lo_to_f32(b.x), acc);
  acc = fmaf(bf16hi_to_f32(a.x), bf16hi_to_f32(b.x), acc);
  acc = fmaf(bf16lo_to_f32(a.y), bf16lo_to_f32(b.y), acc);
  acc = fmaf(bf16hi_to_f32(a.y), bf16hi_to_f32(b.y), acc);
  acc = fmaf(bf16lo_to_f32(a.z), bf16lo_to_f32(b.z), acc);
  acc = fmaf(bf16hi_to_f32(a.z), bf16hi_to_f32(b.z), acc);
  acc = fmaf(bf16lo_to_f32(a.w), bf16lo_to_f32(b.w), acc);
  acc = fmaf(bf16hi_to_f32(a.w), bf16hi_to_f32(b.w), acc);
  return acc;
}

template <int MT>
__host__ __device__ constexpr int gemv_smem_bytes(int K) {
  return MT * K * 2 + MT * 4 + 16;
}

// MT: rows of x held (>= M, power of two). R: output units per warp step. GLU: gate/up units.
template <int MT, int R, bool GLU, bool OUT_F32>
__global__ void __launch_bounds__(kGemvThreads) k_gemv(const uint16_t* __restrict__ x, const uint16_t* __restrict__ w,
                                                      void* __restrict__ y, int M, int K, int n_units, int ldy,
                                                      float eps) {
  constexpr int NR = GLU ? 2 * R : R;  // W* rows per step
  extern __shared__ uint4 smem_v[];
  uint4* xs = smem_v;  // [MT][K/8] chunks
  float* rs = reinterpret_cast<float*>(reinterpret_cast<uint16_t*>(smem_v) + MT * K);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kc = K >> 3;
  {
    // this warp's first group of W* rows into L2 (up to 4 KB a row) while the previous kernel drains
    const int u = (static_cast<int>(blockIdx.x) * (kGemvThreads / 32) + warp) * R + (lane >> 1);
    if (lane < 2 * R && u < n_units && (GLU || (lane & 1) == 0)) {
      const int row = GLU ? ((u >> 4) << 5) + (u & 15) + (lane & 1) * 16 : u;
      bulk_prefetch_l2(w + static_cast<size_t>(row) * K, static_cast<uint32_t>(min(2 * K, 4096) & ~15));
    }
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

  const int groups = (n_units + R - 1) / R;
  for (int gi = blockIdx.x * (kGemvThreads / 32) + warp; gi < groups; gi += gridDim.x * (kGemvThreads / 32)) {
    const uint16_t* rows[NR];
    bool valid[NR];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int u = gi * R + i;
      const bool ok = u < n_units;
      if (GLU) {
        const int gate_row = ((u >> 4) << 5) + (u & 15);
        rows[2 * i] = w + static_cast<size_t>(ok ? gate_row : 0) * K;
        rows[2 * i + 1] = w + static_cast<size_t>(ok ? gate_row + 16 : 0) * K;
        valid[2 * i] = valid[2 * i + 1] = ok;
      } else {
        rows[i] = w + static_cast<size_t>(ok ? u : 0) * K;
        valid[i] = ok;
      }
    }
    float acc[MT][NR];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int j = 0; j < NR; ++j) acc[m][j] = 0.f;

    for (int c0 = lane; c0 < kc; c0 += 32 * kGemvUnroll) {
      uint4 wv[kGemvUnroll][NR];
#pragma unroll
      for (int uu = 0; uu < kGemvUnroll; ++uu) {
        const int c = c0 + uu * 32;
#pragma unroll
        for (int j = 0; j < NR; ++j)
          wv[uu][j] = (c < kc && valid[j]) ? ldg_stream(rows[j] + c * 8) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int uu = 0; uu < kGemvUnroll; ++uu) {
        const int c = c0 + uu * 32;
        if (c < kc) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const uint4 xv = xs[m * kc + c];
#pragma unroll
            for (int j = 0; j < NR; ++j) acc[m][j] = dot8(wv[uu][j], xv, acc[m][j]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int j = 0; j < NR; ++j) acc[m][j] = warp_sum(acc[m][j]);

    // lane l writes unit (l % R) of row (l / R)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
      for (int i = 0; i < R; ++i) {
        if (lane == ((m * R + i) & 31) && m < M) {
          const int u = gi * R + i;
          if (u < n_units) {
            const float r = rs[m];
            float v;
            if (GLU) {
              const float zg = acc[m][2 * i] * r, zu = acc[m][2 * i + 1] * r;
              v = zg / (1.0f + expf(-zg)) * zu;
            } else {
              v = acc[m][i] * r;
            }
            if (OUT_F32)
              static_cast<float*>(y)[static_cast<size_t>(m) * ldy + u] = v;
            else
              static_cast<uint16_t*>(y)[static_cast<size_t>(m) * ldy + u] =
                  static_cast<uint16_t>(pack_bf16x2(v, 0.f) & 0xFFFFu);
          }
        }
      }
    }
  }
}

}  // namespace fn
