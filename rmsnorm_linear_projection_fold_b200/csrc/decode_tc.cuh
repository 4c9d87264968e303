// decode_tc.cuh — decode-sized FlashNorm projections (M <= 16 tokens) on the tensor cores.
//
// Same computation as the prefill kernel, y = (x . W*) * 1/sqrt(mean(x^2) + eps) ("FlashNorm: Fast
// Normalization for Transformers", Abstract, items i and ii), arranged for the memory-bound regime:
// the operands are swapped so that 128 rows of the folded weight W* form the MMA's M side and the
// (at most 16) tokens its N side. Each CTA streams its 128-row slab of W* once through a deep TMA
// ring; the tensor core reduces it against the staged x tiles into a 128 x 16 fp32 accumulator in
// tensor memory, while the same four warps that later run the epilogue sum x^2 per token from the
// staged x tiles (the deferred norm, joined with the MMA by shared-memory barriers).
//
// When there are too few 128-row slabs to occupy the GPU, the contraction is split over K across a
// thread-block cluster of `ksplit` CTAs: every CTA reduces one K range into its own accumulator and
// sum of squares, the partial results are written into the leader CTA's shared memory through the
// cluster's distributed shared memory, and the leader adds them, scales and stores. A CTA whose bounded
// wait gave up sends NaN partial sums, so the outputs they feed are NaN rather than plausible values.
//
// LayerNorm (LN): the same four warps also add up x per token, and the epilogue applies the rank-1 form
// of the fold, y = r (x . W*) - (r mu) colsum(W*) + beta^T W, with mu the token's mean and
// r = 1/sqrt(E[x^2] - mu^2 + eps) (see flashnorm_fold_layernorm).
//
// Warps: 0 = TMA producer, 1 = TMEM allocator + MMA issuer, 2..5 = sum of squares, then epilogue.
#pragma once

#include "sm100.cuh"

namespace fn {

constexpr int kDecRows = 128;              // W* rows per CTA (MMA M)
constexpr int kDecTok = 16;                // token slots (MMA N)
constexpr int kDecWStage = kDecRows * 64 * 2;  // 16 KB
constexpr int kDecXStage = kDecTok * 64 * 2;   // 2 KB
constexpr int kDecThreads = 192;
constexpr int kDecMaxSplit = 4;
// Independent accumulators: the MMAs of a k-block go to four 16-column accumulators in turn, summed in
// the epilogue in a fixed order. MMAs of N = 16 into one accumulator form a dependent chain that runs
// at about one per 150 cycles; four chains overlap in the tensor pipe.
constexpr int kDecAccs = 4;

struct DecodeParams {
  void* y;
  int M;       // tokens (1..16)
  int K;       // d
  int n_rows;  // rows of W* (N, or 2F for GLU)
  int n_out;   // output columns (N, or F)
  int ldy;
  int ksplit;  // CTAs per cluster sharing one slab (1, 2 or 4)
  float eps;
  // LN: fp32 [n_out] column sums of the folded W* and folded bias beta^T W
  const float* ln_colsum = nullptr;
  const float* ln_bias = nullptr;
};

template <int STAGES, int KSPLIT>
__host__ __device__ constexpr int decode_smem_bytes() {
  return 1024 + STAGES * (kDecWStage + kDecXStage) +
         (KSPLIT > 1 ? KSPLIT * (kDecRows * kDecTok + 2 * kDecTok) * 4 : 0) + 1024;
}

template <int STAGES, int KSPLIT, bool GLU, bool OUT_F32, bool LN = false>
__global__ void __launch_bounds__(kDecThreads, 1)
    k_decode_tc(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x, DecodeParams p) {
  static_assert(!(LN && GLU), "LayerNorm is fused into the linear epilogue only");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sW = smem;
  uint8_t* sX = sW + STAGES * kDecWStage;
  float* part_d = reinterpret_cast<float*>(sX + STAGES * kDecXStage);      // [KSPLIT][128][16] (leader)
  float* part_ss = part_d + (KSPLIT > 1 ? KSPLIT * kDecRows * kDecTok : 0);  // [KSPLIT][16]
  float* part_sx = part_ss + (KSPLIT > 1 ? KSPLIT * kDecTok : 0);             // [KSPLIT][16], LN
  uint64_t* full = reinterpret_cast<uint64_t*>(part_sx + (KSPLIT > 1 ? KSPLIT * kDecTok : 0));
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* drain = acc_full + 1;
  float* rs = reinterpret_cast<float*>(drain + 1);  // [16] 1/rms per token
  float* kms = rs + kDecTok;                        // [16] LN: r * mu per token
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(kms + kDecTok);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) >> 5, 0);
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const uint32_t rank = KSPLIT > 1 ? cluster_ctarank() : 0;
  const int slab = static_cast<int>(blockIdx.x) / KSPLIT;
  const int n0 = slab * kDecRows;
  const int num_kb = (p.K + 63) / 64;
  const int kb0 = static_cast<int>((static_cast<long long>(rank) * num_kb) / KSPLIT);
  const int kb1 = static_cast<int>((static_cast<long long>(rank + 1) * num_kb) / KSPLIT);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);  // MMA commit + the four reduction warps
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
    // the first ring's worth of this CTA's W* into L2 while the previous kernel drains
    for (int kb = kb0; kb < kb1 && kb < kb0 + STAGES; ++kb) tma_prefetch_l2_2d(&tm_w, kb * 64, n0);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();  // the previous kernel's outputs (our inputs, or buffers we overwrite) are complete

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
        mbar_arrive_expect_tx(&full[s], kDecWStage + kDecXStage);
        tma_load_2d(sW + s * kDecWStage, &tm_w, &full[s], kb * 64, n0);
        tma_load_2d(sX + s * kDecXStage, &tm_x, &full[s], kb * 64, 0);
        ++issued;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      grid_dep_launch();  // all loads issued: the next kernel may be scheduled onto SMs as they free up
      if (ok) {
        // Wait for the release of the last use of every stage, so that no arrival on this CTA's barriers
        // (an MMA commit completes asynchronously) is still in flight when the CTA exits.
        for (int i = 0; i < STAGES; ++i) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) break;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        const int pending = issued < STAGES ? issued : STAGES;
        for (int i = 1; i <= pending; ++i) {
          int st = s - i;
          uint32_t pp = ph;
          if (st < 0) {
            st += STAGES;
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
      const uint32_t idesc = make_idesc_bf16(kDecRows, kDecTok);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[s], ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_u32(sW + s * kDecWStage);
        const uint32_t b_addr = smem_u32(sX + s * kDecXStage);
#pragma unroll
        for (int k = 0; k < 4; ++k)  // MMA k of every k-block into accumulator k
          tc_mma_bf16(tmem_base + static_cast<uint32_t>(k * kDecTok), make_sdesc_sw128(a_addr + k * 32),
                      make_sdesc_sw128(b_addr + k * 32), idesc, kb != kb0 ? 1u : 0u);
        tc_commit(&empty[s]);
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      // An empty K range (more CTAs than k-blocks) leaves the accumulator unwritten: the epilogue
      // then treats it as zero.
      tc_commit(ok ? acc_full : drain);
      if (!ok) {
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // -------------------------------------------------------------- sum of squares, then epilogue
    const int t = static_cast<int>(threadIdx.x) - 64;  // 0..127
    const int tok = t >> 3, chunk = t & 7;             // one 16-byte chunk of one token's row per stage
    const int q = warp & 3;                            // TMEM lane quarter
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    float ss = 0.f, sx = 0.f;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(&full[s], ph, abort_flag)) {
        ok = false;
        break;
      }
      const uint4 w = *reinterpret_cast<const uint4*>(sX + s * kDecXStage + tok * 128 + chunk * 16);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = bf16lo_to_f32(ws[i]), hi = bf16hi_to_f32(ws[i]);
        ss = fmaf(lo, lo, ss);
        ss = fmaf(hi, hi, ss);
        if (LN) sx += lo + hi;
      }
      fence_proxy_async_smem();  // the reads above come before the TMA refill this arrival permits
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == STAGES) {
        s = 0;
        ph ^= 1u;
      }
    }
    // A wait that gave up leaves this thread's part of the sum incomplete: it contributes NaN instead,
    // so every output that depends on it is written as NaN (the status word reports the timeout).
    const float kNaN = __int_as_float(0x7fc00000);
    if (!ok) ss = kNaN;
    // the eight threads of a token are eight consecutive lanes
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (LN) sx += __shfl_xor_sync(0xffffffffu, sx, o);
    }

    float v[kDecTok];
    const bool have_acc = ok && kb1 > kb0;
    if (ok && have_acc) ok = mbar_wait(acc_full, 0, abort_flag);
    if (have_acc && ok) {
      tc_fence_after_sync();
      uint32_t r0[16], r1[16], r2[16], r3[16];
      const uint32_t lanes = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      tmem_ld16(lanes, r0);
      tmem_ld16(lanes + kDecTok, r1);
      tmem_ld16(lanes + 2 * kDecTok, r2);
      tmem_ld16(lanes + 3 * kDecTok, r3);
      tmem_ld_wait();
      reg_fence16(r0);
      reg_fence16(r1);
      reg_fence16(r2);
      reg_fence16(r3);
#pragma unroll
      for (int j = 0; j < kDecTok; ++j)
        v[j] = (__uint_as_float(r0[j]) + __uint_as_float(r1[j])) + (__uint_as_float(r2[j]) + __uint_as_float(r3[j]));
    } else {
      // an empty K range (more CTAs than k-blocks) contributes zero; a failed wait contributes NaN
#pragma unroll
      for (int j = 0; j < kDecTok; ++j) v[j] = ok ? 0.f : kNaN;
    }
    const int row = q * 32 + lane;  // W* row within the slab held by this thread
    if (KSPLIT > 1) {
      if (rank != 0) {
        const uint32_t dst = dsmem_addr(part_d + (rank * kDecRows + row) * kDecTok, 0);
#pragma unroll
        for (int j = 0; j < kDecTok; j += 4) dsmem_st_v4(dst + j * 4, v[j], v[j + 1], v[j + 2], v[j + 3]);
        if (chunk == 0) dsmem_st_f32(dsmem_addr(part_ss + rank * kDecTok + tok, 0), ss);
        if (LN && chunk == 0) dsmem_st_f32(dsmem_addr(part_sx + rank * kDecTok + tok, 0), sx);
      }
    }
    if (KSPLIT > 1) cluster_sync_all();  // every thread of the cluster, also warps 0 and 1 (below)
    if (rank == 0) {
      if (KSPLIT > 1) {
        for (int rr = 1; rr < KSPLIT; ++rr) {
#pragma unroll
          for (int j = 0; j < kDecTok; ++j) v[j] += part_d[(rr * kDecRows + row) * kDecTok + j];
          if (chunk == 0) ss += part_ss[rr * kDecTok + tok];
          if (LN && chunk == 0) sx += part_sx[rr * kDecTok + tok];
        }
      }
      if (chunk == 0) {
        if (LN) {
          // biased variance E[x^2] - mu^2, clamped at 0 against rounding; eps inside the root
          const float mu = sx / static_cast<float>(p.K);
          const float var = fmaxf(ss / static_cast<float>(p.K) - mu * mu, 0.0f);
          rs[tok] = 1.0f / sqrtf(var + p.eps);
          kms[tok] = rs[tok] * mu;
        } else {
          rs[tok] = 1.0f / sqrtf(ss / static_cast<float>(p.K) + p.eps);
        }
      }
      named_bar_sync(1, 128);
      {
        if (!GLU) {
          const int n = n0 + row;
          float cn = 0.f, bn = 0.f;
          if (LN && n < p.n_out) cn = __ldg(p.ln_colsum + n), bn = __ldg(p.ln_bias + n);
#pragma unroll
          for (int m = 0; m < kDecTok; ++m) {
            if (m >= p.M) break;
            const float o = LN ? fmaf(v[m], rs[m], fmaf(-kms[m], cn, bn)) : v[m] * rs[m];
            if (n < p.n_out) {
              if (OUT_F32)
                static_cast<float*>(p.y)[static_cast<size_t>(m) * p.ldy + n] = o;
              else
                static_cast<uint16_t*>(p.y)[static_cast<size_t>(m) * p.ldy + n] =
                    static_cast<uint16_t>(pack_bf16x2(o, 0.f) & 0xFFFFu);
            }
          }
        } else {
          // rows 32b + j (gate) and 32b + 16 + j (up) are lanes j and j + 16 of one warp
          const int col = ((n0 + q * 32) >> 1) + (lane & 15);
#pragma unroll
          for (int m = 0; m < kDecTok; ++m) {
            if (m >= p.M) break;
            const float up = __shfl_down_sync(0xffffffffu, v[m], 16);
            if (lane < 16 && col < p.n_out) {
              const float zg = v[m] * rs[m], zu = up * rs[m];
              float e, sg;
              asm("ex2.approx.f32 %0, %1;" : "=f"(e) : "f"(-zg * 1.4426950408889634f));
              asm("rcp.approx.f32 %0, %1;" : "=f"(sg) : "f"(1.0f + e));
              const float o = zg * sg * zu;
              if (OUT_F32)
                static_cast<float*>(p.y)[static_cast<size_t>(m) * p.ldy + col] = o;
              else
                static_cast<uint16_t*>(p.y)[static_cast<size_t>(m) * p.ldy + col] =
                    static_cast<uint16_t>(pack_bf16x2(o, 0.f) & 0xFFFFu);
            }
          }
        }
      }
    }
  }
  if (KSPLIT > 1 && warp < 2) cluster_sync_all();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, 64);
}

}  // namespace fn
