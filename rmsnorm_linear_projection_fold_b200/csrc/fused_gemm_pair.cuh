// fused_gemm_pair.cuh — the FlashNorm prefill kernel on CTA pairs (tcgen05 cta_group::2).
//
// Same computation and warp roles as fused_gemm.cuh (deferred normalisation of "FlashNorm: Fast
// Normalization for Transformers", Abstract, item ii: x . W* on the tensor cores, sum of x^2 per row
// on a separate warpgroup from the same staged x tiles, joined in the epilogue), but two CTAs of a
// cluster share each MMA of M = 256 rows:
//   * each CTA stages its own 128 rows of x and HALF of the tile's W* rows (split along N), so the W*
//     bytes a CTA moves per MMA are halved and a stage shrinks from 48 KB to 32 KB (six stages fit);
//   * the leader CTA (cluster rank 0) issues the pair MMA; both CTAs' TMA loads report to the
//     leader's stage barrier, and the leader's commits arrive on both CTAs' barriers (commit
//     multicast; every TMA load is an ordinary single-CTA fetch);
//   * each CTA's tensor memory holds the accumulator of its own 128 rows, read by its own epilogue;
//   * each CTA's sum-of-squares warps read only their own x tile, and only on a row block's first tile
//     in this pair's tile range (later tiles of the row block reuse its 1/rms). On those stage uses the
//     leader forwards "stage landed" (xfull) to both CTAs once the whole pair stage is in, and the
//     stage is refilled only after the MMA's commit (empty) AND the CTA's own reduction warps
//     (xempty) have released it, the explicit join of the 1-SM kernel. On every other use the MMA's
//     commit alone releases the stage and the reduction warps take no part: no waits or arrivals on
//     the MMA issuer's or the producer's path. Producer, MMA issuer and reduction warps all derive
//     which uses are read from the same tile sequence, so their phase counts agree stage by stage;
//   * the epilogue stages each warp's 32 rows x 64 bytes of output in swizzled shared memory and writes
//     them back row-contiguously (8 rows x 64 bytes per warp store) instead of every lane storing its
//     own row (32 cache lines per warp store, which made the epilogue as long as a short-K tile).
#pragma once

#include "fused_gemm.cuh"

namespace fn {

constexpr int kPairStages = 6;
constexpr int kPairStageOutBytes = 32 * 64;  // per epilogue warp: 32 rows x 64 bytes of y
constexpr int kPairBHalfRows = 128;                       // W* rows per CTA per stage, at most
constexpr int kPairBStage = kPairBHalfRows * kBK * 2;     // 16 KB

template <int STAGES>
__host__ __device__ constexpr int gemm_pair_smem_bytes() {
  return 1024 + STAGES * (kAStageBytes + kPairBStage) + 8 * kPairStageOutBytes + 4096;
}

// Output columns per staged chunk (64 bytes of a row). The pair kernel's tile width is chosen so that
// every tile's output columns are a whole number of chunks.
__host__ __device__ constexpr int pair_chunk_cols(bool out_f32) { return out_f32 ? 16 : 32; }

// p.num_m_tiles counts 256-row pair tiles; p.bn is the pair tile width (W* rows), each CTA holding bn/2.
// Schedule. CTA pairs form groups of p.group (1 or 2); the pairs of a group work on the same W* column
// tiles at the same time, each in its own row block, so that a W* tile fetched from HBM by one is found
// in L2 by the other (W* is streamed once per group instead of once per pair: the Llama-7B SwiGLU
// weights, 180 MB, do not fit in L2). A "group tile" is one column tile of a band of p.group row
// blocks; groups take contiguous ranges of group tiles (band-major), so a pair stays in one row block
// for most of its range and reads that block's x tiles for its sum of squares only once. When the
// group tiles leave a short last wave, those past p.num_main are each split into two halves of bn/2
// columns, one half per group: with 688 tiles on 74 pairs (Llama-7B SwiGLU, 2048 tokens) every pair
// runs 9 full tiles and at most one half tile, 9.5 tile times instead of 10. tm_w loads the W* rows of
// a full tile (bn/2 per CTA), tm_w2 those of a half tile (bn/4 per CTA).
template <int STAGES, int EPI, bool SCALE, bool OUT_F32>
__global__ void __launch_bounds__(gemm_threads(EPI, SCALE), 1)
    k_fused_gemm_pair(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_w2, GemmParams p) {
  constexpr bool LN = EPI == EPI_LN;
  static_assert(!LN || SCALE, "the LayerNorm epilogue needs the mean and variance warps");
  constexpr int kSsWarps = SCALE ? 4 : 0;
  constexpr int kEpiWarps = gemm_epi_warps(EPI);
  constexpr int kEpiFirst = 2, kSsFirst = 2 + kEpiWarps;
  static_assert(EPI != EPI_POSTNORM, "the pair kernel has no per-head post-norm epilogue");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kAStageBytes;
  uint8_t* sOut = sB + STAGES * kPairBStage;  // [8 epilogue warps][32 rows x 64 B], swizzled
  uint8_t* tail = sOut + 8 * kPairStageOutBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);  // used in the leader
  uint64_t* empty = full + STAGES;
  uint64_t* xfull = empty + STAGES;                     // "x tile of this stage has landed" (reduction)
  uint64_t* xempty = xfull + STAGES;                    // "reduction warps are done with this stage"
  uint64_t* acc_full = xempty + STAGES;                 // [2]
  uint64_t* acc_empty = acc_full + 2;                   // [2], used in the leader
  uint64_t* ss_full = acc_empty + 2;                    // [2]
  uint64_t* ss_empty = ss_full + 2;                     // [2]
  uint64_t* drain = ss_empty + 2;                       // [1]
  float* rinv = reinterpret_cast<float*>(drain + 1);    // [2][128]
  float* kmu = rinv + 2 * kBM;                          // [2][128], LayerNorm: r * mean(x)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(kmu + 2 * kBM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) >> 5, 0);
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);  // the leader's expect-tx arrival covers both CTAs' bytes
      mbar_init(&empty[s], 1);  // the MMA's commit (multicast to both CTAs)
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], kSsWarps > 0 ? kSsWarps : 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);
      mbar_init(&ss_full[b], kBM);
      mbar_init(&ss_empty[b], 32 * kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_w2);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before either touches the other's
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();  // the previous kernel's outputs (our inputs, or buffers we overwrite) are complete

  const int G = p.group;
  const int cl = static_cast<int>(blockIdx.x) >> 1;        // CTA pair
  const int grp = cl / G, kg = cl % G;                    // group, and this pair's row block in the band
  const int ngrp = (static_cast<int>(gridDim.x) >> 1) / G;
  const int num_gtiles = (p.num_m_tiles / G) * p.num_n_tiles;
  const int t_begin = static_cast<int>(static_cast<long long>(grp) * p.num_main / ngrp);
  const int t_end = static_cast<int>(static_cast<long long>(grp + 1) * p.num_main / ngrp);
  const int num_halves = 2 * (num_gtiles - p.num_main);
  // the half tiles go to the last groups, whose ranges end nearest to them (fewer fresh row blocks)
  const int half_id = grp - (ngrp - num_halves);
  const int n_items = (t_end - t_begin) + (half_id >= 0 ? 1 : 0);
  const int num_kb = (p.K + kBK - 1) / kBK;
  const int bn = p.bn;
  // Item i of this pair: its row block, first W* row and width (full tiles first, then a half tile).
  auto tile_at = [&](int i, int& mt, int& n0, int& width) {
    if (i < t_end - t_begin) {
      const int u = t_begin + i;
      mt = (u / p.num_n_tiles) * G + kg;
      n0 = (u % p.num_n_tiles) * bn;
      width = bn;
    } else {
      const int u = p.num_main + (half_id >> 1);
      mt = (u / p.num_n_tiles) * G + kg;
      n0 = (u % p.num_n_tiles) * bn + (half_id & 1) * (bn / 2);
      width = bn / 2;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      // per CTA; the leader announces the whole pair stage, the peer's loads only complete on it
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      uint32_t x_read = 0;  // bit s: the current use of stage s is read by the reduction warps
      uint32_t x_ph = 0;    // bit s: parity of the next xempty phase of stage s
      int last_m = -1;
      for (int i = 0; i < n_items && ok; ++i) {
        int mt, n0t, width;
        tile_at(i, mt, n0t, width);
        const bool fresh = SCALE && mt != last_m;
        last_m = mt;
        const int m0 = mt * (2 * kBM) + static_cast<int>(rank) * kBM;
        const int n0 = n0t + static_cast<int>(rank) * (width / 2);
        const uint32_t stage_bytes = static_cast<uint32_t>(kAStageBytes + (width / 2) * kBK * 2);
        const CUtensorMap* map_w = width == bn ? &tm_w : &tm_w2;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_cluster(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (SCALE && ((x_read >> s) & 1u)) {  // the previous use was also read by the reduction warps
            if (!mbar_wait(&xempty[s], (x_ph >> s) & 1u, abort_flag)) {
              ok = false;
              break;
            }
            x_ph ^= 1u << s;
          }
          x_read = fresh ? (x_read | (1u << s)) : (x_read & ~(1u << s));
          const uint32_t leader_full = dsmem_addr(&full[s], 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * stage_bytes);
          tma_load_2d_pair(sA + s * kAStageBytes, &tm_x, leader_full, kb * kBK, m0);
          tma_load_2d_pair(sB + s * kPairBStage, map_w, leader_full, kb * kBK, n0);
          ++issued;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      grid_dep_launch();  // all loads issued: the next kernel may be scheduled onto SMs as they free up
      if (ok) {
        // Wait for the release of the last use of every stage, so that no arrival on this CTA's barriers
        // (an MMA commit completes asynchronously) is still in flight when the CTA exits.
        for (int i = 0; i < STAGES; ++i) {
          if (!mbar_wait_cluster(&empty[s], ph ^ 1u, abort_flag)) break;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok && leader) {
        // Gave up: let the pair's copies still in flight land (bounded) before shared memory goes.
        const int pending = issued < STAGES ? issued : STAGES;
        for (int i = 1; i <= pending; ++i) {
          int st = s - i;
          uint32_t pp = ph;
          if (st < 0) {
            st += STAGES;
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
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      int last_m = -1;
      for (int i = 0; i < n_items && ok; ++i) {
        int mt, n0t, width;
        tile_at(i, mt, n0t, width);
        const uint32_t idesc = make_idesc_bf16(2 * kBM, width);
        const bool fresh = SCALE && mt != last_m;
        last_m = mt;
        if (!mbar_wait_cluster(&acc_empty[acc], acc_ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_cluster(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          if (fresh) {  // both CTAs' reduction warps may read their x tiles now
            mbar_arrive(&xfull[s]);
            mbar_arrive_remote(dsmem_addr(&xfull[s], 1));
          }
          const uint32_t a_addr = smem_u32(sA + s * kAStageBytes);
          const uint32_t b_addr = smem_u32(sB + s * kPairBStage);
#pragma unroll
          for (int k = 0; k < kBK / kMmaK; ++k)
            tc_mma_bf16_pair(d_tmem, make_sdesc_sw128(a_addr + k * kMmaK * 2),
                             make_sdesc_sw128(b_addr + k * kMmaK * 2), idesc, (kb | k) != 0 ? 1u : 0u);
          tc_commit_pair_mc(&empty[s], 0x3);  // frees stage s in both CTAs once read
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(&acc_full[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1u;
      }
      if (!ok) {
        tc_commit_pair_mc(drain, 0x1);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp < kSsFirst) {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int hh = (warp - kEpiFirst) >> 2;  // which of the two warps on this lane quarter
    const int row_in_tile = q * 32 + lane;
    const uint32_t leader_acc_empty0 = dsmem_addr(&acc_empty[0], 0);
    const uint32_t leader_acc_empty1 = dsmem_addr(&acc_empty[1], 0);
    int acc = 0;
    uint32_t acc_ph = 0;
    int sb = 0;
    uint32_t sb_ph = 0;
    for (int i = 0; i < n_items; ++i) {
      int mt, n0t, width;
      tile_at(i, mt, n0t, width);
      if (!mbar_wait_cluster(&acc_full[acc], acc_ph, abort_flag)) break;
      tc_fence_after_sync();
      float r = 1.0f, km = 0.0f;
      if (SCALE) {
        if (!mbar_wait(&ss_full[sb], sb_ph, abort_flag)) break;
        r = rinv[sb * kBM + row_in_tile];
        if (LN) km = kmu[sb * kBM + row_in_tile];
        mbar_arrive(&ss_empty[sb]);
        sb ^= 1;
        if (sb == 0) sb_ph ^= 1u;
      }
      const GluRow kr = glu_row(r);
      // rows of this warp's lane quarter in y, and its staging buffer
      const int qrow0 = mt * (2 * kBM) + static_cast<int>(rank) * kBM + q * 32;
      uint8_t* stage_out = sOut + (warp - kEpiFirst) * kPairStageOutBytes;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * 256);
      constexpr int CC = pair_chunk_cols(OUT_F32);
      constexpr int kEsz = OUT_F32 ? 4 : 2;
      const int ocols = EPI == EPI_GLU ? width / 2 : width;
      const int ocol0 = EPI == EPI_GLU ? n0t / 2 : n0t;
      // 16-byte piece j (0..3) of row r sits at r*64 + ((j ^ (r >> 1)) & 3) * 16: conflict-free both for
      // a quarter-warp writing one piece of eight rows and for one reading two whole rows.
      auto put16 = [&](int j, uint4 v) {
        *reinterpret_cast<uint4*>(stage_out + lane * 64 + (((j ^ (lane >> 1)) & 3) << 4)) = v;
      };
      // The two warps of a lane quarter take alternate chunks; which one starts alternates from tile to
      // tile, so an odd chunk count does not always land on the same warp.
      for (int ch = (hh + i) & 1; ch * CC < ocols && ocol0 + ch * CC < p.n_out; ch += 2) {
        if (EPI == EPI_LINEAR || LN) {
          // CC accumulator columns -> CC outputs (4 pieces of 16 bytes): the deferred scale r, and for
          // LayerNorm also the rank-1 mean correction and the folded bias, y = r acc - (r mu) colsum + bias
          const int col = ocol0 + ch * CC;
          float cq[CC], bq[CC];
          if (LN) {
#pragma unroll
            for (int k = 0; k < CC / 4; ++k) {
              float4 c4 = make_float4(0.f, 0.f, 0.f, 0.f), b4 = c4;
              if (col + 4 * k < p.n_out) {  // n_out % 8 == 0: a group of 4 columns is wholly in or out
                c4 = __ldg(reinterpret_cast<const float4*>(p.ln_colsum + col) + k);
                b4 = __ldg(reinterpret_cast<const float4*>(p.ln_bias + col) + k);
              }
              cq[4 * k] = c4.x, cq[4 * k + 1] = c4.y, cq[4 * k + 2] = c4.z, cq[4 * k + 3] = c4.w;
              bq[4 * k] = b4.x, bq[4 * k + 1] = b4.y, bq[4 * k + 2] = b4.z, bq[4 * k + 3] = b4.w;
            }
          }
          uint32_t v0[16], v1[16];
          tmem_ld16(t_row + ch * CC, v0);
          if constexpr (CC == 32) tmem_ld16(t_row + ch * CC + 16, v1);
          tmem_ld_wait();
          reg_fence16(v0);
          if constexpr (CC == 32) reg_fence16(v1);
          float o[CC];
#pragma unroll
          for (int jj = 0; jj < CC; ++jj) {
            const float a = __uint_as_float(jj < 16 ? v0[jj & 15] : v1[jj & 15]);
            o[jj] = LN ? fmaf(a, r, fmaf(-km, cq[jj], bq[jj])) : a * r;
          }
          if (OUT_F32) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
              put16(jj, make_uint4(__float_as_uint(o[4 * jj]), __float_as_uint(o[4 * jj + 1]),
                                   __float_as_uint(o[4 * jj + 2]), __float_as_uint(o[4 * jj + 3])));
          } else {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
              put16(jj, make_uint4(pack_bf16x2(o[8 * jj], o[8 * jj + 1]), pack_bf16x2(o[8 * jj + 2], o[8 * jj + 3]),
                                   pack_bf16x2(o[8 * jj + 4], o[8 * jj + 5]), pack_bf16x2(o[8 * jj + 6], o[8 * jj + 7])));
          }
        } else {
          // CC output columns = CC/16 (gate 16, up 16) pairs of accumulator columns, all loaded from tensor
          // memory before one wait, so that the load latency is paid once per chunk
          uint32_t gt[CC / 16][16], up[CC / 16][16];
#pragma unroll
          for (int b = 0; b < CC / 16; ++b) {
            const int acol = 2 * (ch * CC) + 32 * b;
            tmem_ld16(t_row + acol, gt[b]);
            tmem_ld16(t_row + acol + 16, up[b]);
          }
          tmem_ld_wait();
#pragma unroll
          for (int b = 0; b < CC / 16; ++b) {
            reg_fence16(gt[b]);
            reg_fence16(up[b]);
          }
#pragma unroll
          for (int b = 0; b < CC / 16; ++b) {
            float o[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              o[j] = swiglu_deferred(__uint_as_float(gt[b][j]), __uint_as_float(up[b][j]), kr);
            if (OUT_F32) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                put16(j, make_uint4(__float_as_uint(o[4 * j]), __float_as_uint(o[4 * j + 1]),
                                    __float_as_uint(o[4 * j + 2]), __float_as_uint(o[4 * j + 3])));
            } else {
#pragma unroll
              for (int j = 0; j < 2; ++j)
                put16(2 * b + j, make_uint4(pack_bf16x2(o[8 * j], o[8 * j + 1]), pack_bf16x2(o[8 * j + 2], o[8 * j + 3]),
                                            pack_bf16x2(o[8 * j + 4], o[8 * j + 5]), pack_bf16x2(o[8 * j + 6], o[8 * j + 7])));
            }
          }
        }
        __syncwarp();
        // write back: lane l copies piece (l & 3) of rows 8i + (l >> 2); a 16-byte piece lies wholly inside
        // or wholly past column n_out (n_out is a multiple of 8).
        const int seg = lane & 3;
        const int col = ocol0 + ch * CC + seg * (16 / kEsz);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rr = 8 * i + (lane >> 2);
          const uint4 v = *reinterpret_cast<const uint4*>(stage_out + rr * 64 + (((seg ^ (rr >> 1)) & 3) << 4));
          const int row = qrow0 + rr;
          if (row < p.M && col < p.n_out)
            *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.y) +
                                      (static_cast<size_t>(row) * p.ldy + col) * kEsz) = v;
        }
        __syncwarp();  // the staging buffer is read before the next chunk overwrites it
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&acc_empty[acc]);
        else
          mbar_arrive_remote(acc == 0 ? leader_acc_empty0 : leader_acc_empty1);
      }
      acc ^= 1;
      if (acc == 0) acc_ph ^= 1u;
    }
  } else if (SCALE) {
    // ------------------------------------------------------------------ sum of squares (both CTAs)
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int s = 0;
    uint32_t x_ph = 0;  // bit s: parity of the next xfull phase of stage s (one phase per use read)
    int sb = 0;
    uint32_t sb_ph = 0;
    int last_m = -1;
    float r_row = 0.0f, km_row = 0.0f;
    bool ok = true;
    for (int i = 0; i < n_items && ok; ++i) {
      int mt, n0t, width;
      tile_at(i, mt, n0t, width);
      const bool fresh = mt != last_m;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      float s0 = 0.f, s1 = 0.f;  // LayerNorm: sum of x
      if (!fresh) {
        // this row block's 1/rms is known: the tile's stage uses pass without us
        s = (s + num_kb) % STAGES;
      }
      for (int kb = 0; fresh && kb < num_kb; ++kb) {
        // Every use read here is waited for in order, so this warp is never more than one xfull phase
        // behind and the parity wait is unambiguous.
        if (!mbar_wait_cluster(&xfull[s], (x_ph >> s) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        x_ph ^= 1u << s;
        const uint8_t* line = sA + s * kAStageBytes + row_in_tile * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(line + (((c ^ lane) & 7) << 4));
          float f;
          f = bf16lo_to_f32(w.x); a0 = fmaf(f, f, a0); if (LN) s0 += f;
          f = bf16hi_to_f32(w.x); a1 = fmaf(f, f, a1); if (LN) s1 += f;
          f = bf16lo_to_f32(w.y); a2 = fmaf(f, f, a2); if (LN) s0 += f;
          f = bf16hi_to_f32(w.y); a3 = fmaf(f, f, a3); if (LN) s1 += f;
          f = bf16lo_to_f32(w.z); a0 = fmaf(f, f, a0); if (LN) s0 += f;
          f = bf16hi_to_f32(w.z); a1 = fmaf(f, f, a1); if (LN) s1 += f;
          f = bf16lo_to_f32(w.w); a2 = fmaf(f, f, a2); if (LN) s0 += f;
          f = bf16hi_to_f32(w.w); a3 = fmaf(f, f, a3); if (LN) s1 += f;
        }
        fence_proxy_async_smem();  // reads above before the TMA refill our arrival permits
        __syncwarp();
        if (lane == 0) mbar_arrive(&xempty[s]);
        if (++s == STAGES) s = 0;
      }
      if (!ok) break;
      if (fresh) {
        const float ss = (a0 + a1) + (a2 + a3);
        if (LN) {
          // LayerNorm: biased variance E[x^2] - mean^2 (clamped at 0 against rounding), eps inside the root
          const float mu = (s0 + s1) / static_cast<float>(p.K);
          const float var = fmaxf(ss / static_cast<float>(p.K) - mu * mu, 0.0f);
          r_row = 1.0f / sqrtf(var + p.eps);
          km_row = r_row * mu;
        } else {
          r_row = 1.0f / sqrtf(ss / static_cast<float>(p.K) + p.eps);
        }
        last_m = mt;
      }
      if (!mbar_wait(&ss_empty[sb], sb_ph ^ 1u, abort_flag)) break;
      rinv[sb * kBM + row_in_tile] = r_row;
      if (LN) kmu[sb * kBM + row_in_tile] = km_row;
      mbar_arrive(&ss_full[sb]);
      sb ^= 1;
      if (sb == 0) sb_ph ^= 1u;
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while the other may still signal its barriers
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace fn
