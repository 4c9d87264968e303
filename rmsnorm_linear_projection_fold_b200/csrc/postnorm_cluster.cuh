// postnorm_cluster.cuh — redundant-norm removal for wide heads (head_dim in {384, 512} here, e.g.
// a 512-wide MLA latent): y = u / sqrt(mean_head(u^2) + eps2) * g2 with u = x . W*, the first
// RMSNorm dropped and its gain folded into W* ("FlashNorm: Fast Normalization for Transformers",
// Abstract: a linear layer between two RMSNorms lets the first one go, by scale invariance).
//
// One 128-row tile of one head is computed by a thread-block cluster of CN x KS CTAs:
//   * CN = head_dim / 128 column slices: each CTA owns 128 output columns of the head, so a row's
//     norm needs the other slices' partial sums of squares, exchanged through distributed shared
//     memory (DSMEM);
//   * KS (1 or 2) K-ranges: each CTA contracts one range of d into its own 128 x 128 fp32
//     accumulator in tensor memory; the ks = 1 CTA parks its accumulator in its own shared memory and
//     pushes it with one bulk DSMEM copy into the (by then idle) pipeline buffers of the ks = 0 CTA
//     of its slice, which adds it to its own.
// The CTA is kept under half an SM's shared memory, so that two fit on an SM and every cluster of a
// launch can be resident at once (a cluster that does not fit would run as a second wave).
// A wide head therefore spreads over CN * KS SMs instead of one, which is what keeps the GPU busy
// when there are only M / 128 row tiles.
//
// Warps: 0 = TMA producer, 1 = TMEM allocator + MMA issuer, 2..5 = epilogue (one row per thread).
#pragma once

#include "sm100.cuh"

namespace fn {

constexpr int kPnCols = 128;                     // columns per CTA
constexpr int kPnStageBytes = 128 * 64 * 2 * 2;  // x tile + W* tile, 32 KB
constexpr int kPnStages = 3;
constexpr int kPnThreads = 192;
constexpr int kPnPStride = kPnCols + 4;          // padded row stride (floats) of a parked accumulator
constexpr uint32_t kPnParkBytes = 128u * kPnPStride * 4u;
static_assert(kPnParkBytes <= static_cast<uint32_t>(kPnStages * kPnStageBytes), "parked tile must fit the stages");

struct PostnormClusterParams {
  void* y;
  const uint16_t* g2;  // bf16 [head_dim]
  int M, K, N, head_dim;
  int num_m_tiles;
  int cn, ks;  // column slices and K ranges per cluster
  float eps2;
};

__host__ __device__ constexpr int postnorm_cluster_smem_bytes() {
  return 1024 + kPnStages * kPnStageBytes + 4 * kPnCols * 4 /* ss exchange */ + 512 * 4 /* g2 */ + 1024;
}

template <bool OUT_F32>
__global__ void __launch_bounds__(kPnThreads, 1)
    k_postnorm_cluster(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                       PostnormClusterParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* stages = smem;                                                  // [kPnStages][x 16K | W 16K]
  float* parked = reinterpret_cast<float*>(smem);                          // reuses the stages afterwards
  float* ssx = reinterpret_cast<float*>(smem + kPnStages * kPnStageBytes);  // [4][128] partial sums
  float* g2s = ssx + 4 * kPnCols;                                          // [512]
  uint64_t* full = reinterpret_cast<uint64_t*>(g2s + 512);
  uint64_t* empty = full + kPnStages;
  uint64_t* acc_full = empty + kPnStages;
  uint64_t* drain = acc_full + 1;
  uint64_t* recv = drain + 1;  // the K partner's parked accumulator has landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recv + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) >> 5, 0);
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const int csize = p.cn * p.ks;
  const uint32_t rank = cluster_ctarank();
  const int cn = static_cast<int>(rank) % p.cn;
  const int ks = static_cast<int>(rank) / p.cn;
  const int cluster = static_cast<int>(blockIdx.x) / csize;
  const int mt = cluster % p.num_m_tiles;
  const int head = cluster / p.num_m_tiles;
  const int m0 = mt * 128;
  const int col0 = head * p.head_dim + cn * kPnCols;  // first output column / W* row of this CTA
  const int num_kb = (p.K + 63) / 64;
  const int kb0 = static_cast<int>((static_cast<long long>(ks) * num_kb) / p.ks);
  const int kb1 = static_cast<int>((static_cast<long long>(ks + 1) * num_kb) / p.ks);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPnStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init(recv, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kPnCols);
    tmem_relinquish();
  }
  grid_dep_wait();  // the previous kernel's outputs (our inputs, or buffers we overwrite) are complete
  for (int i = static_cast<int>(threadIdx.x); i < p.head_dim; i += kPnThreads)
    g2s[i] = __uint_as_float(static_cast<uint32_t>(p.g2[i]) << 16);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* st = stages + s * kPnStageBytes;
        mbar_arrive_expect_tx(&full[s], kPnStageBytes);
        tma_load_2d(st, &tm_x, &full[s], kb * 64, m0);
        tma_load_2d(st + kPnStageBytes / 2, &tm_w, &full[s], kb * 64, col0);
        ++issued;
        if (++s == kPnStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      grid_dep_launch();  // all loads issued: the next kernel may be scheduled onto SMs as they free up
      if (ok) {
        // Wait for the release of the last use of every stage, so that no arrival on this CTA's barriers
        // (an MMA commit completes asynchronously) is still in flight when the CTA exits.
        for (int i = 0; i < kPnStages; ++i) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) break;
          if (++s == kPnStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        const int pending = issued < kPnStages ? issued : kPnStages;
        for (int i = 1; i <= pending; ++i) {
          int st = s - i;
          uint32_t pp = ph;
          if (st < 0) {
            st += kPnStages;
            pp ^= 1u;
          }
          const unsigned long long t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[st], pp) && globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(128, kPnCols);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[s], ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_u32(stages + s * kPnStageBytes);
        const uint32_t b_addr = a_addr + kPnStageBytes / 2;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_bf16(tmem_base, make_sdesc_sw128(a_addr + k * 32), make_sdesc_sw128(b_addr + k * 32), idesc,
                      (kb != kb0 || k != 0) ? 1u : 0u);
        tc_commit(&empty[s]);
        if (++s == kPnStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      tc_commit(ok ? acc_full : drain);
      if (!ok) {
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue, one row per thread
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const bool have_acc = kb1 > kb0;
    bool ok = true;
    if (have_acc) ok = mbar_wait(acc_full, 0, abort_flag);
    if (have_acc) tc_fence_after_sync();
    // The pipeline is drained once the accumulator is complete (every MMA has read its stage), so the
    // stage buffers are free: the ks = 1 CTA parks its partial there, the ks = 0 CTA receives it there.
    const int et = static_cast<int>(threadIdx.x) - 64;  // 0..127 over the epilogue warps
    if (ks > 0) {
      for (int c = 0; c < kPnCols; c += 16) {
        uint32_t v[16];
        if (have_acc && ok) {
          tmem_ld16(t_row + c, v);
          tmem_ld_wait();
          reg_fence16(v);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0u;
        }
        float4* dst = reinterpret_cast<float4*>(parked + row * kPnPStride + c);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                               __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
      }
      fence_proxy_async_smem();  // the bulk copy (async proxy) reads what these stores wrote
    } else if (p.ks > 1 && et == 0) {
      mbar_arrive_expect_tx(recv, kPnParkBytes);
    }
    cluster_sync_all();  // (1) partners parked; receivers' buffers free and expecting
    if (ks > 0 && et == 0) {
      const uint32_t dst_rank = static_cast<uint32_t>(cn);  // the ks = 0 CTA of this slice
      bulk_push_dsmem(dsmem_addr(parked, dst_rank), parked, kPnParkBytes, dsmem_addr(recv, dst_rank));
    }
    bool got = true;
    if (ks == 0 && p.ks > 1) got = mbar_wait(recv, 0, abort_flag);

    // u for 16 columns of this row: own accumulator plus the received partial of the K partner
    auto load_u = [&](int c, float (&u)[16]) {
      if (have_acc && ok) {
        uint32_t v[16];
        tmem_ld16(t_row + c, v);
        tmem_ld_wait();
        reg_fence16(v);
#pragma unroll
        for (int j = 0; j < 16; ++j) u[j] = __uint_as_float(v[j]);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) u[j] = 0.f;
      }
      if (p.ks > 1 && got) {
        const float4* src = reinterpret_cast<const float4*>(parked + row * kPnPStride + c);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 a = src[j];
          u[4 * j] += a.x;
          u[4 * j + 1] += a.y;
          u[4 * j + 2] += a.z;
          u[4 * j + 3] += a.w;
        }
      }
    };

    if (ks == 0) {
      float ss = 0.f;
      for (int c = 0; c < kPnCols; c += 16) {
        float u[16];
        load_u(c, u);
#pragma unroll
        for (int j = 0; j < 16; ++j) ss = fmaf(u[j], u[j], ss);
      }
      // hand this slice's partial sum of squares to every slice of the head
      for (int o = 0; o < p.cn; ++o) dsmem_st_f32(dsmem_addr(ssx + cn * kPnCols + row, static_cast<uint32_t>(o)), ss);
    }
    cluster_sync_all();  // (2) partial sums of squares exchanged

    if (ks == 0 && ok && got) {
      float ss = 0.f;
      for (int o = 0; o < p.cn; ++o) ss += ssx[o * kPnCols + row];
      const float r2 = 1.0f / sqrtf(ss / static_cast<float>(p.head_dim) + p.eps2);
      const int grow = m0 + row;
      for (int c = 0; c < kPnCols; c += 16) {
        float u[16];
        load_u(c, u);
        float o[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j] = u[j] * r2 * g2s[cn * kPnCols + c + j];
        if (grow < p.M) {
          if (OUT_F32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.y) + static_cast<size_t>(grow) * p.N + col0 + c);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.y) + static_cast<size_t>(grow) * p.N + col0 + c);
            dst[0] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                pack_bf16x2(o[6], o[7]));
            dst[1] = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]), pack_bf16x2(o[12], o[13]),
                                pack_bf16x2(o[14], o[15]));
          }
        }
      }
    }
    cluster_sync_all();  // (3) partners keep their parked partials until every reader is done
  }
  if (warp < 2) {
    cluster_sync_all();
    cluster_sync_all();
    cluster_sync_all();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, kPnCols);
}

}  // namespace fn
