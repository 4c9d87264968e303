// postnorm_pair.cuh — redundant-norm removal for wide heads (256 < head_dim <= 512, e.g. the
// 512-wide MLA latent) on CTA pairs: y = u / sqrt(mean_head(u^2) + eps2) * g2 with u = x . W*, the
// first RMSNorm dropped and its gain folded into W* ("FlashNorm: Fast Normalization for
// Transformers", Abstract: a linear layer between two RMSNorms lets the first one go, by the scale
// invariance of RMS).
//
// A wide head has few row tiles (M / 256 of them), so each 256-row tile of one head is spread over a
// thread-block cluster of 2 x NP x KS CTAs:
//   * CTA pairs share each MMA (tcgen05 cta_group::2, M = 256): every CTA stages its own 128 rows of
//     x and half of the pair's W* rows, so each SM moves 32 KB per 64-deep k-block for a 128 x 256
//     block of the product (twice the work per byte of a 1-CTA 128 x 128 tile);
//   * NP = 2 column halves of the head, one pair each (MMA N = head_dim / 2);
//   * KS = 1 to 4 ranges of the contraction dimension d, one pair each.
// After the contraction the KS pairs of a column half hold partial sums of the same 256 x hd/2 block.
// They reduce-scatter it through distributed shared memory: the block's columns are cut into KS
// slices of whole 16-column chunks (hd / (2 KS) wide, or nearly), every CTA sends the slices it does not
// own into the (by then idle) pipeline buffers of their owners and adds the ones it receives to its own
// slice, in a fixed order of K ranges (deterministic). Each CTA then holds the complete u for 128 rows
// x its slice's columns; the per-row sums of squares over those columns go to every CTA of the cluster
// that holds the same rows, and each CTA scales and stores its own slice. No partial result goes
// through global memory.
//
// Warps: 0 = TMA producer, 1 = TMEM allocator + pair MMA issuer (leader CTA of the pair),
// 2..9 = epilogue (two warps per tensor-memory lane quarter, splitting a slice's columns).
#pragma once

#include "sm100.cuh"

namespace fn {

constexpr int kPpStages = 6;
constexpr int kPpAStage = 128 * 64 * 2;  // 16 KB: 128 rows of x, 64 k-values
constexpr int kPpBStage = 128 * 64 * 2;  // room for up to 128 W* rows (a quarter of a 512-wide head)
constexpr int kPpThreads = 64 + 8 * 32;
constexpr int kPpNP = 2;                 // column halves of a head
constexpr int kPpMaxKS = 4;
constexpr int kPpMaxHead = 512;

struct PostnormPairParams {
  void* y;
  const uint16_t* g2;  // bf16 [head_dim]
  int M, K, N, head_dim;
  int num_m_tiles;     // 256-row tiles
  int ks;              // K ranges per cluster (1 to kPpMaxKS); cluster = 2 * kPpNP * ks CTAs
  float eps2;
};

__host__ __device__ constexpr int postnorm_pair_smem_bytes() {
  return 1024 + kPpStages * (kPpAStage + kPpBStage) + kPpNP * kPpMaxKS * 2 * 128 * 4 /* ss partials */ +
         kPpMaxHead * 4 /* g2 */ + 512 /* barriers */;
}

// Row stride (floats) of a received slice: its width plus one 16-byte pad, so that eight consecutive
// rows written with 16-byte stores land in distinct bank groups.
__host__ __device__ constexpr int pp_slice_stride(int w) { return w + 4; }

// First column of slice k of nw columns cut into ks slices of whole 16-column chunks (the last takes
// the remainder: 256 in three is 80, 80, 96).
__host__ __device__ constexpr int pp_slice_begin(int k, int nw, int ks) { return k >= ks ? nw : (k * nw / ks) / 16 * 16; }

template <bool OUT_F32>
__global__ void __launch_bounds__(kPpThreads, 1)
    k_postnorm_pair(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    PostnormPairParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPpStages * kPpAStage;
  float* recv = reinterpret_cast<float*>(smem);  // reuses the stages once every MMA has read them
  float* ssx = reinterpret_cast<float*>(smem + kPpStages * (kPpAStage + kPpBStage));  // [NP*KS*2][128]
  float* g2s = ssx + kPpNP * kPpMaxKS * 2 * 128;                                      // [head_dim]
  uint64_t* full = reinterpret_cast<uint64_t*>(g2s + kPpMaxHead);  // used in the leader
  uint64_t* empty = full + kPpStages;
  uint64_t* acc_full = empty + kPpStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) >> 5, 0);
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const int KS = p.ks;
  const int csize = 2 * kPpNP * KS;
  const uint32_t rank = cluster_ctarank();
  const int half = static_cast<int>(rank & 1u);          // which 128 rows of the pair tile
  const uint32_t lead = rank & ~1u;                      // the pair's leader CTA
  const bool leader = half == 0;
  const int np = static_cast<int>(rank >> 1) % kPpNP;    // column half of the head
  const int ks = static_cast<int>(rank >> 1) / kPpNP;    // K range
  const int cluster = static_cast<int>(blockIdx.x) / csize;
  const int mt = cluster % p.num_m_tiles;
  const int head = cluster / p.num_m_tiles;
  const int hd = p.head_dim;
  const int nw = hd / 2;          // MMA N: the pair's columns
  const int brows = hd / 4;       // W* rows this CTA stages
  // the slice of the pair's columns this CTA finishes, and the widest slice (the receive slots' width)
  const int c_own = pp_slice_begin(ks, nw, KS);
  const int w = pp_slice_begin(ks + 1, nw, KS) - c_own;
  int w_max = 0;
  for (int k = 0; k < KS; ++k) w_max = max(w_max, pp_slice_begin(k + 1, nw, KS) - pp_slice_begin(k, nw, KS));
  const int sstr = pp_slice_stride(w_max);
  const int m0 = mt * 256 + half * 128;
  const int col_pair = head * hd + np * nw;  // first output column / W* row of the pair
  const int num_kb = (p.K + 63) / 64;
  const int kb0 = static_cast<int>((static_cast<long long>(ks) * num_kb) / KS);
  const int kb1 = static_cast<int>((static_cast<long long>(ks + 1) * num_kb) / KS);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPpStages; ++s) {
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
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 256);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // every CTA's barriers exist before any CTA touches another's
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();  // the previous kernel's outputs (our inputs, or buffers we overwrite) are complete
  for (int i = static_cast<int>(threadIdx.x); i < hd; i += kPpThreads)
    g2s[i] = __uint_as_float(static_cast<uint32_t>(p.g2[i]) << 16);
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t stage_bytes = static_cast<uint32_t>(kPpAStage + brows * 64 * 2);
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_cluster(&empty[s], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t leader_full = dsmem_addr(&full[s], lead);
        if (leader) mbar_arrive_expect_tx(&full[s], 2 * stage_bytes);
        tma_load_2d_pair(sA + s * kPpAStage, &tm_x, leader_full, kb * 64, m0);
        tma_load_2d_pair(sB + s * kPpBStage, &tm_w, leader_full, kb * 64, col_pair + half * brows);
        ++issued;
        if (++s == kPpStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      grid_dep_launch();  // all loads issued: the next kernel may be scheduled onto SMs as they free up
      if (ok) {
        // wait for the release of every stage's last use: no commit arrival is in flight at exit
        for (int i = 0; i < kPpStages; ++i) {
          if (!mbar_wait_cluster(&empty[s], ph ^ 1u, abort_flag)) break;
          if (++s == kPpStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      } else if (leader) {
        // gave up: let the pair's copies still in flight land (bounded) before shared memory goes
        const int pending = issued < kPpStages ? issued : kPpStages;
        for (int i = 1; i <= pending; ++i) {
          int st = s - i;
          uint32_t pp = ph;
          if (st < 0) {
            st += kPpStages;
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
      const uint16_t mask = static_cast<uint16_t>(3u << lead);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_cluster(&full[s], ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_u32(sA + s * kPpAStage);
        const uint32_t b_addr = smem_u32(sB + s * kPpBStage);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_bf16_pair(tmem_base, make_sdesc_sw128(a_addr + k * 32), make_sdesc_sw128(b_addr + k * 32), idesc,
                           (kb != kb0 || k != 0) ? 1u : 0u);
        tc_commit_pair_mc(&empty[s], mask);  // frees stage s in both CTAs once read
        if (++s == kPpStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (ok) {
        tc_commit_pair_mc(acc_full, mask);
      } else {
        tc_commit_pair_mc(drain, static_cast<uint16_t>(1u << lead));
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  }

  // ------------------------------------------------------------------ epilogue (warps 2..9)
  const bool epi = warp >= 2;
  const int q = warp & 3;                    // tensor-memory lane quarter
  const int h2 = (warp - 2) >> 2;            // which of the two warps on this quarter
  const int row = q * 32 + lane;             // row within this CTA's 128
  const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
  const int nchunks = w / 16;
  bool ok = true;
  if (epi) {
    ok = mbar_wait_cluster(acc_full, 0, abort_flag);
    if (ok) tc_fence_after_sync();
  }
  // (1) every CTA's contraction is complete, so every CTA's stage buffers are idle
  cluster_sync_all();

  // 16 columns [c, c+16) of this row's partial accumulator (zero if the contraction gave up)
  auto load_acc = [&](int c, float (&u)[16]) {
    if (ok) {
      uint32_t v[16];
      tmem_ld16(t_row + static_cast<uint32_t>(c), v);
      tmem_ld_wait();
      reg_fence16(v);
#pragma unroll
      for (int j = 0; j < 16; ++j) u[j] = __uint_as_float(v[j]);
    } else {
      const float nan = __int_as_float(0x7fc00000);
#pragma unroll
      for (int j = 0; j < 16; ++j) u[j] = nan;  // a failed wait poisons what it feeds
    }
  };

  if (epi && KS > 1) {
    // send the slices this CTA does not own to their owners: slot (source K range, skipping the owner's)
    for (int d = 1; d < KS; ++d) {
      const int dst_ks = (ks + d) % KS;
      const int slot = ks < dst_ks ? ks : ks - 1;
      const uint32_t dst_rank = static_cast<uint32_t>((dst_ks * kPpNP + np) * 2 + half);
      const uint32_t dst = dsmem_addr(recv + (slot * 128 + row) * sstr, dst_rank);
      const int c_dst = pp_slice_begin(dst_ks, nw, KS);
      const int n_dst = (pp_slice_begin(dst_ks + 1, nw, KS) - c_dst) / 16;
      for (int ch = h2; ch < n_dst; ch += 2) {
        float u[16];
        load_acc(c_dst + ch * 16, u);
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          dsmem_st_v4(dst + static_cast<uint32_t>((ch * 16 + j) * 4), u[j], u[j + 1], u[j + 2], u[j + 3]);
      }
    }
  }
  // (2) every slice has reached its owner
  cluster_sync_all();

  // u for 16 columns of this CTA's own slice: the K ranges' partial sums added in range order
  auto slice_u = [&](int ch, float (&u)[16]) {
#pragma unroll
    for (int j = 0; j < 16; ++j) u[j] = 0.f;
    for (int k = 0; k < KS; ++k) {
      float part[16];
      if (k == ks) {
        load_acc(c_own + ch * 16, part);
      } else {
        const int slot = k < ks ? k : k - 1;
        const float4* src = reinterpret_cast<const float4*>(recv + (slot * 128 + row) * sstr + ch * 16);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 a = src[j];
          part[4 * j] = a.x, part[4 * j + 1] = a.y, part[4 * j + 2] = a.z, part[4 * j + 3] = a.w;
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) u[j] += part[j];
    }
  };

  if (epi) {
    float ss = 0.f;
    for (int ch = h2; ch < nchunks; ch += 2) {
      float u[16];
      slice_u(ch, u);
#pragma unroll
      for (int j = 0; j < 16; ++j) ss = fmaf(u[j], u[j], ss);
    }
    // this warp's partial sum of squares of the row goes to every CTA that holds the same rows
    const int slot = ((ks * kPpNP + np) * 2 + h2) * 128 + row;
    for (int k = 0; k < KS; ++k)
      for (int n = 0; n < kPpNP; ++n)
        dsmem_st_f32(dsmem_addr(ssx + slot, static_cast<uint32_t>((k * kPpNP + n) * 2 + half)), ss);
  }
  // (3) the partial sums of squares are exchanged
  cluster_sync_all();

  if (epi) {
    float ss = 0.f;
    for (int i = 0; i < kPpNP * KS * 2; ++i) ss += ssx[i * 128 + row];  // fixed order: deterministic
    const float r2 = 1.0f / sqrtf(ss / static_cast<float>(hd) + p.eps2);
    const int grow = m0 + row;
    for (int ch = h2; ch < nchunks; ch += 2) {
      float u[16];
      slice_u(ch, u);
      const int lc = np * nw + c_own + ch * 16;  // column within the head
      float o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = u[j] * r2 * g2s[lc + j];
      if (grow < p.M) {
        const size_t off = static_cast<size_t>(grow) * p.N + head * hd + lc;
        if (OUT_F32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.y) + off);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.y) + off);
          dst[0] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                              pack_bf16x2(o[6], o[7]));
          dst[1] = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]), pack_bf16x2(o[12], o[13]),
                              pack_bf16x2(o[14], o[15]));
        }
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while another may still signal its barriers or read its memory
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 256);
}

}  // namespace fn
