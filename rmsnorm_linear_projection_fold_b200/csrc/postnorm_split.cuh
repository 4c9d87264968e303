// postnorm_split.cuh — redundant-norm removal for wide heads (256 < head_dim <= 512, e.g. the 512-wide
// MLA latent) with the contraction spread over independent CTA pairs: y = u / sqrt(mean_head(u^2) + eps2)
// * g2 with u = x . W*, the first RMSNorm dropped and its gain folded into W* ("FlashNorm: Fast
// Normalization for Transformers", Abstract: a linear layer between two RMSNorms lets the first one go).
//
// The cluster kernel (postnorm_pair.cuh) keeps every partial sum on chip, but one cluster has to hold
// all K ranges and both column halves of a 256-row tile, and few clusters that large are resident at
// once (2048 rows of one 512-wide head run on 64 SMs). Here each CTA pair is its own cluster of two:
//   k_postnorm_split_gemm: one pair (tcgen05 cta_group::2, M = 256) per 256-row tile, head, column half
//     (MMA N = head_dim / 2) and range of the contraction dimension d. It writes the fp32 partial product
//     of its 128 rows x head_dim / 2 columns over its K range to a caller-provided workspace,
//     ws[k][m][n] (one [M, N] plane per K range), with TMA stores;
//   k_postnorm_finalize: one warp per (row, head) adds the K ranges' partials in range order (the same
//     sums whatever the schedule: deterministic), takes the head's mean square and writes
//     y = u * 1/sqrt(mean(u^2) + eps2) * g2.
// The second kernel is launched with programmatic dependent launch: it is scheduled as the first drains
// and waits (griddepcontrol.wait) for the first's completion before it reads the workspace.
//
// Warps of the GEMM: 0 = TMA producer, 1 = TMEM allocator + pair MMA issuer (leader CTA),
// 2..9 = epilogue (two warps per tensor-memory lane quarter, splitting the columns).
#pragma once

#include "sm100.cuh"

namespace fn {

constexpr int kPsStages = 6;
constexpr int kPsAStage = 128 * 64 * 2;  // 16 KB: 128 rows of x, 64 k-values
constexpr int kPsBStage = 128 * 64 * 2;  // up to 128 W* rows (a quarter of a 512-wide head)
constexpr int kPsThreads = 64 + 8 * 32;
constexpr int kPsMaxKS = 8;              // K ranges
constexpr int kPfWarps = 8;              // warps per CTA of the finalize kernel
constexpr int kPsBoxBytes = 32 * 128 * 4;  // one TMA store box of the partial product: 32 columns x 128 rows

struct PostnormSplitParams {
  int M, K, N, head_dim;
  int num_m_tiles;  // 256-row tiles
  int heads;        // N / head_dim
  int ks;           // K ranges
};

struct PostnormFinalizeParams {
  const float* ws;     // fp32 [ks][M][N]
  const uint16_t* g2;  // bf16 [head_dim]
  void* y;
  int M, N, head_dim, heads, ks;
  float eps2;
};

__host__ __device__ constexpr int postnorm_split_smem_bytes() {
  return 1024 + kPsStages * (kPsAStage + kPsBStage) + 256 /* barriers */;
}

__global__ void __launch_bounds__(kPsThreads, 1)
    k_postnorm_split_gemm(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                          const __grid_constant__ CUtensorMap tm_ws, PostnormSplitParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPsStages * kPsAStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPsStages * (kPsAStage + kPsBStage));  // leader's
  uint64_t* empty = full + kPsStages;
  uint64_t* acc_full = empty + kPsStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) >> 5, 0);
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const int half = static_cast<int>(cluster_ctarank() & 1u);  // which 128 rows of the pair tile
  const bool leader = half == 0;
  // pair index -> (row tile, column half, head, K range), row tiles fastest
  int rest = static_cast<int>(blockIdx.x) / 2;
  const int mt = rest % p.num_m_tiles;
  rest /= p.num_m_tiles;
  const int np = rest & 1;
  rest >>= 1;
  const int head = rest % p.heads;
  const int kr = rest / p.heads;
  const int hd = p.head_dim;
  const int nw = hd / 2;     // MMA N: the pair's columns
  const int brows = hd / 4;  // W* rows this CTA stages
  const int m0 = mt * 256 + half * 128;
  const int col_pair = head * hd + np * nw;  // first output column / W* row of the pair
  const int num_kb = (p.K + 63) / 64;
  const int kb0 = static_cast<int>((static_cast<long long>(kr) * num_kb) / p.ks);
  const int kb1 = static_cast<int>((static_cast<long long>(kr + 1) * num_kb) / p.ks);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPsStages; ++s) {
      mbar_init(&full[s], 1);   // the leader's expect-tx arrival covers both CTAs' bytes
      mbar_init(&empty[s], 1);  // the pair MMA's commit, multicast to both CTAs
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_ws);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 256);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before either touches the other's
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();  // the previous kernel (which may read the workspace we overwrite) has completed

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t stage_bytes = static_cast<uint32_t>(kPsAStage + brows * 64 * 2);
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_cluster(&empty[s], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t leader_full = dsmem_addr(&full[s], 0);
        if (leader) mbar_arrive_expect_tx(&full[s], 2 * stage_bytes);
        tma_load_2d_pair(sA + s * kPsAStage, &tm_x, leader_full, kb * 64, m0);
        tma_load_2d_pair(sB + s * kPsBStage, &tm_w, leader_full, kb * 64, col_pair + half * brows);
        ++issued;
        if (++s == kPsStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      grid_dep_launch();  // all loads issued: the finalize kernel may be scheduled as SMs free up
      if (ok) {
        // wait for the release of every stage's last use: no commit arrival is in flight at exit
        for (int i = 0; i < kPsStages; ++i) {
          if (!mbar_wait_cluster(&empty[s], ph ^ 1u, abort_flag)) break;
          if (++s == kPsStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      } else if (leader) {
        // gave up: let the pair's copies still in flight land (bounded) before shared memory goes
        const int pending = issued < kPsStages ? issued : kPsStages;
        for (int i = 1; i <= pending; ++i) {
          int st = s - i;
          uint32_t pp = ph;
          if (st < 0) {
            st += kPsStages;
            pp ^= 1u;
          }
          const unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait_cluster(&full[st], pp) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ pair MMA issuer (leader)
    if (lane == 0 && leader) {
      const uint32_t idesc = make_idesc_bf16(256, nw);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_cluster(&full[s], ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_u32(sA + s * kPsAStage);
        const uint32_t b_addr = smem_u32(sB + s * kPsBStage);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_bf16_pair(tmem_base, make_sdesc_sw128(a_addr + k * 32), make_sdesc_sw128(b_addr + k * 32), idesc,
                           (kb != kb0 || k != 0) ? 1u : 0u);
        tc_commit_pair_mc(&empty[s], 3u);  // frees stage s in both CTAs once read
        if (++s == kPsStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (ok) {
        tc_commit_pair_mc(acc_full, 3u);
      } else {
        tc_commit_pair_mc(drain, 1u);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;          // tensor-memory lane quarter
    const int h2 = (warp - 2) >> 2;  // which of the two warps on this quarter
    const int row = q * 32 + lane;   // row within this CTA's 128
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    // warp-uniform: a lane that saw the accumulator late must not leave the others in a collective load
    const bool ok = __all_sync(0xffffffffu, mbar_wait_cluster(acc_full, 0, abort_flag) ? 1 : 0) != 0;
    if (ok) tc_fence_after_sync();
    // The partial product leaves through TMA stores of 32-column x 128-row boxes staged in the pipeline
    // buffers (idle once the accumulator is complete) in the 128-byte swizzled layout: row r's 16-byte
    // chunk c sits at r * 128 + ((c ^ (r & 7)) * 16), so the 32 rows of a warp's stores hit distinct
    // banks, and each box row goes out as one full 128-byte line.
    const uint32_t r7 = static_cast<uint32_t>(row & 7);
    const int nchunks = nw / 16;  // a multiple of 2: the split path takes head_dim % 64 == 0
    // round i: chunks 4i .. 4i+3 (this warp: ch and ch + 2), i.e. boxes 2i and 2i + 1
    for (int ch = h2; ch < nchunks; ch += 4) {
      const bool two = ch + 2 < nchunks;  // the same for both warps of a quarter: nchunks is even
      uint32_t v[2][16];
      if (ok) {
        tmem_ld16(t_row + static_cast<uint32_t>(ch * 16), v[0]);
        if (two) tmem_ld16(t_row + static_cast<uint32_t>((ch + 2) * 16), v[1]);
        tmem_ld_wait();
        reg_fence16(v[0]);
        reg_fence16(v[1]);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[0][j] = v[1][j] = 0x7fc00000u;  // a failed wait poisons the result
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (c == 1 && !two) break;
        const int cc = ch + 2 * c;  // chunk: box cc / 2, 16-byte chunks (cc & 1) * 4 .. + 3 of its row
        const uint32_t box = smem_u32(smem) + static_cast<uint32_t>((cc >> 1) * kPsBoxBytes + row * 128);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t chunk = (static_cast<uint32_t>((cc & 1) * 4 + j) ^ r7) * 16u;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(box + chunk), "r"(v[c][4 * j]),
                       "r"(v[c][4 * j + 1]), "r"(v[c][4 * j + 2]), "r"(v[c][4 * j + 3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();   // the generic-proxy writes, visible to the TMA engine
      named_bar_sync(1, 8 * 32);  // all eight epilogue warps wrote this round's boxes
      if (warp == 2 && lane == 0 && m0 < p.M) {  // rows past M are clipped by the store itself
        const int b0 = (ch - h2) >> 1;
        for (int b = b0; b < b0 + (two ? 2 : 1); ++b)
          tma_store_3d(&tm_ws, smem + b * kPsBoxBytes, col_pair + 32 * b, m0, kr);
        tma_store_commit();
      }
    }
    if (warp == 2 && lane == 0) tma_store_wait_all();  // written before the kernel (and its smem) ends
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the other may still signal its barriers
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 256);
}

// One warp per (row, head). Lane l holds the head's columns 4l + 128j .. 4l + 128j + 3 (j = 0..3), so
// each load and store of a warp covers 512 (fp32) or 256 (bf16) contiguous bytes. KS (the number of K
// ranges) is a compile-time constant so that all KS x 4 loads of a row are issued before the first add:
// one round trip to L2 per row instead of one per K range.
template <int KS, bool OUT_F32>
__global__ void __launch_bounds__(kPfWarps * 32, 2) k_postnorm_finalize(PostnormFinalizeParams p) {
  const int warp = static_cast<int>(threadIdx.x) >> 5;
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const int hd = p.head_dim;
  // g2 is read before the wait. This kernel is scheduled only once every CTA of the GEMM has issued its
  // loads, which each does after its own wait on the kernel before it: whatever wrote g2 has completed.
  float g[16];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int c = 4 * lane + 128 * j + t;
      g[4 * j + t] = c < hd ? __uint_as_float(static_cast<uint32_t>(p.g2[c]) << 16) : 0.f;
    }
  grid_dep_wait();    // the GEMM's partial products are complete and visible
  grid_dep_launch();  // the next kernel may start its prologue; it waits for this one before any access
  const long long items = static_cast<long long>(p.M) * p.heads;
  const size_t plane = static_cast<size_t>(p.M) * p.N;
  for (long long it = static_cast<long long>(blockIdx.x) * kPfWarps + warp; it < items;
       it += static_cast<long long>(gridDim.x) * kPfWarps) {
    const int m = static_cast<int>(it / p.heads);
    const int h = static_cast<int>(it % p.heads);
    const size_t off = static_cast<size_t>(m) * p.N + static_cast<size_t>(h) * hd;
    // every K range's partials first (independent loads in flight), then their sum in range order
    float4 part[KS][4];
#pragma unroll
    for (int k = 0; k < KS; ++k)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 4 * lane + 128 * j;
        part[k][j] = c < hd ? __ldcg(reinterpret_cast<const float4*>(p.ws + k * plane + off + c))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    float u[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float4 a = part[0][j];
#pragma unroll
      for (int k = 1; k < KS; ++k)
        a = make_float4(a.x + part[k][j].x, a.y + part[k][j].y, a.z + part[k][j].z, a.w + part[k][j].w);
      u[4 * j] = a.x, u[4 * j + 1] = a.y, u[4 * j + 2] = a.z, u[4 * j + 3] = a.w;
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) ss = fmaf(u[j], u[j], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r2 = 1.0f / sqrtf(ss / static_cast<float>(hd) + p.eps2);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = 4 * lane + 128 * j;
      if (c >= hd) continue;
      const float o0 = u[4 * j] * r2 * g[4 * j], o1 = u[4 * j + 1] * r2 * g[4 * j + 1];
      const float o2 = u[4 * j + 2] * r2 * g[4 * j + 2], o3 = u[4 * j + 3] * r2 * g[4 * j + 3];
      if (OUT_F32) {
        *reinterpret_cast<float4*>(static_cast<float*>(p.y) + off + c) = make_float4(o0, o1, o2, o3);
      } else {
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.y) + off + c) =
            make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
      }
    }
  }
}

}  // namespace fn
