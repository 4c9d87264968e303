// fused_gemm.cuh — the FlashNorm prefill kernel for sm_100a.
//
// One persistent kernel computes, per 128-row tile of x and per tile of W* columns,
//     acc = x . W*                      (tcgen05 MMA, fp32 accumulator in tensor memory)
//     ss  = sum_k x[m,k]^2              (a separate warpgroup, CUDA cores, same shared-memory x tiles)
//     y   = epilogue(acc, 1/sqrt(ss/d + eps))
// which is the deferred normalisation of "FlashNorm: Fast Normalization for Transformers" (Abstract,
// item ii): the RMS reduction no longer blocks the matrix multiplication; the two run concurrently on
// different warps and meet at the epilogue. The pages' own design ran them on two CUDA streams and
// found a race when the join between them was implicit (talk summary, "Implementation and
// Concurrency Challenges"); here the join is explicit and on-chip:
//   * each shared-memory stage is released only after BOTH of its consumers are done with it (the
//     MMA's commit and one arrival per sum-of-squares warp), so TMA never overwrites an x tile that
//     the reduction has not read. The reduction reads with ordinary (generic-proxy) loads while TMA
//     writes through the async proxy, so each reduction warp also issues a proxy fence before its
//     arrival; without it the refill could overtake the reads, and the rows' 1/rms picked up parts
//     of the next k-block (seen on tiles after a CTA's first: the stale-buffer race of the pages,
//     moved on-chip);
//   * the epilogue waits on both the accumulator-ready barrier and the rms-ready barrier of the
//     same tile before it scales anything.
//
// Warp roles:
//   warp 0      TMA producer: x tile [128 x 64] and W* tile [bn x 64] per k-block into a smem ring
//   warp 1      TMEM allocator; one lane issues tcgen05.mma and the commits
//   epilogue    8 warps (4 for POSTNORM): tcgen05.ld from TMEM, scale / SwiGLU / per-head RMSNorm,
//               global stores. Warp w may only read TMEM lanes 32*(w%4)..+31, so two warps share
//               each lane quarter and split the tile's columns between them.
//   reduction   4 warps, sum of squares of x per row (only when the deferred scale is used)
//
// Epilogues: LINEAR  y = r * acc
//            GLU     y = silu(r * acc_gate) * (r * acc_up)   (gate/up interleaved in blocks of 16 cols)
//            POSTNORM (pre-norm elided) y = acc / sqrt(mean_head(acc^2) + eps2) * g2
#pragma once

#include "sm100.cuh"

namespace fn {

constexpr int kBM = 128;                     // rows of x per tile (TMEM lanes)
constexpr int kBK = 64;                      // k per stage: 64 bf16 = one 128-byte swizzle row
constexpr int kAStageBytes = kBM * kBK * 2;  // 16 KB
constexpr int kMmaK = 16;                    // k of one kind::f16 MMA
constexpr uint32_t kTmemCols = 512;          // whole tensor memory of the SM (one CTA per SM)

// EPI_LN: LayerNorm -> linear (CTA-pair kernel only): y = r (x . W*) - (r mu) colsum(W*) + beta^T W.
enum EpiKind { EPI_LINEAR = 0, EPI_GLU = 1, EPI_POSTNORM = 2, EPI_LN = 3 };

struct GemmParams {
  void* y;                // output [M, ldy] (bf16 or fp32)
  const uint16_t* g2;     // POSTNORM: bf16 gain [head_dim]
  int M;                  // rows of x / y
  int K;                  // contraction length d
  int n_out;              // output columns (N, or F for GLU)
  int ldy;                // output row stride, elements
  int bn;                 // accumulator tile width (W* rows per tile)
  int head_dim;           // POSTNORM head width
  int num_m_tiles;
  int num_n_tiles;
  float eps;              // eps of the deferred norm (LINEAR/GLU) or eps2 (POSTNORM)
  // POSTNORM with RoPE on the first n_rope_heads heads of a row (rope_cs == nullptr: none)
  const float* rope_cs = nullptr;  // (cos, sin) fp32 [max_pos][head_dim / 2][2]
  const int* positions = nullptr;  // int32 [M], position of each row
  int n_rope_heads = 0;
  int max_pos = 0;
  // EPI_LN: fp32 [n_out] column sums of the folded W* and folded bias beta^T W
  const float* ln_colsum = nullptr;
  const float* ln_bias = nullptr;
  // CTA-pair kernel: pairs work in groups of `group` (1 or 2) on bands of `group` row blocks; group
  // tiles 0 .. num_main-1 are full width, the rest are split in two halves
  int group = 1;
  int num_main = 0;
};

template <int MAX_BN>
struct GemmSmem {
  static constexpr int kBStageBytes = MAX_BN * kBK * 2;
};

// Epilogue warps: two per TMEM lane quarter, except the per-head post-norm, whose row norms need
// all of a head's columns in one thread.
__host__ __device__ constexpr int gemm_epi_warps(int epi) { return epi == 2 /* EPI_POSTNORM */ ? 4 : 8; }
__host__ __device__ constexpr int gemm_threads(int epi, bool scale) {
  return 64 + 32 * gemm_epi_warps(epi) + (scale ? 128 : 0);
}

template <int MAX_BN, int STAGES>
__host__ __device__ constexpr int gemm_smem_bytes() {
  return 1024 /* alignment slack */ + STAGES * (kAStageBytes + MAX_BN * kBK * 2) + 4096 /* barriers etc. */;
}

// The SwiGLU output with the deferred scale r = 1/rms applied to gate and up:
//   silu(r g) (r u) = g u r^2 sigmoid(r g) = g u / ((1 + 2^(-r log2(e) g)) / r^2).
// With the per-row constants c = -r log2(e) and q = 1/r^2 (= mean(x^2) + eps) this is one multiply,
// one SFU exp, one fused multiply-add, one SFU reciprocal and two multiplies per output: two issue
// slots fewer than scaling gate and up first, in an epilogue whose speed is set by its instruction
// count. sigmoid(t) = 1 / (1 + 2^(-t log2(e))) with both the exp and the reciprocal on the
// special-function unit (flush-to-zero forms, one instruction each; relative error ~1e-6). Limits:
// r g -> -inf gives 2^+inf = inf and an output of 0; r g -> +inf gives g u r^2.
struct GluRow {
  float c;  // -r * log2(e)
  float q;  // 1 / r^2
};

__device__ __forceinline__ GluRow glu_row(float r) {
  GluRow k;
  k.c = -r * 1.4426950408889634f;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(k.q) : "f"(r * r));
  return k;
}

__device__ __forceinline__ float swiglu_deferred(float g, float u, GluRow k) {
  float e, s;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(g * k.c));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(s) : "f"(fmaf(e, k.q, k.q)));
  return (g * u) * s;
}

// Store 16 consecutive output values of one row (bf16 or fp32), masking whole 8-column groups.
template <bool OUT_F32>
__device__ __forceinline__ void store16(void* y, int ldy, int row, int col, int n_out, const float (&v)[16]) {
  if (OUT_F32) {
    float* p = static_cast<float*>(y) + static_cast<size_t>(row) * ldy + col;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (col + 8 * h + 8 <= n_out) {
        float4* q = reinterpret_cast<float4*>(p + 8 * h);
        q[0] = make_float4(v[8 * h + 0], v[8 * h + 1], v[8 * h + 2], v[8 * h + 3]);
        q[1] = make_float4(v[8 * h + 4], v[8 * h + 5], v[8 * h + 6], v[8 * h + 7]);
      }
    }
  } else {
    uint16_t* p = static_cast<uint16_t*>(y) + static_cast<size_t>(row) * ldy + col;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (col + 8 * h + 8 <= n_out) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * h + 0], v[8 * h + 1]);
        w.y = pack_bf16x2(v[8 * h + 2], v[8 * h + 3]);
        w.z = pack_bf16x2(v[8 * h + 4], v[8 * h + 5]);
        w.w = pack_bf16x2(v[8 * h + 6], v[8 * h + 7]);
        *reinterpret_cast<uint4*>(p + 8 * h) = w;
      }
    }
  }
}

template <int MAX_BN, int STAGES, int EPI, bool SCALE, bool OUT_F32>
__global__ void __launch_bounds__(gemm_threads(EPI, SCALE), 1)
    k_fused_gemm(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, GemmParams p) {
  constexpr int kAccBufs = (MAX_BN <= 256) ? 2 : 1;
  constexpr int kBStage = MAX_BN * kBK * 2;
  constexpr int kSsWarps = SCALE ? 4 : 0;
  constexpr int kEpiWarps = gemm_epi_warps(EPI);
  constexpr int kEpiFirst = 2, kSsFirst = 2 + kEpiWarps;

  extern __shared__ uint8_t smem_raw[];
  // Stage buffers must sit on 1024-byte boundaries (the 128-byte swizzle repeats every 8 rows).
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kAStageBytes;
  uint8_t* tail = sB + STAGES * kBStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* ss_full = acc_empty + 2;     // [2]
  uint64_t* ss_empty = ss_full + 2;      // [2]
  uint64_t* drain = ss_empty + 2;        // [1]
  float* rinv = reinterpret_cast<float*>(drain + 1);  // [2][128]
  float* g2s = rinv + 2 * kBM;                        // [512]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(g2s + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) >> 5, 0);
  const int lane = static_cast<int>(threadIdx.x) & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kSsWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
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
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();  // the previous kernel's outputs (our inputs, or buffers we overwrite) are complete

  // Tile schedule: the tiles are numbered row-block-major (t -> m = t / num_n, n = t % num_n) and each
  // CTA takes one contiguous, balanced range of them. Consecutive tiles of a CTA then mostly share
  // their 128 rows of x, so the reduction warps compute a row's 1/rms once per row block and reuse
  // it, and the x tiles they reload stay hot in L2.
  const int num_tiles = p.num_m_tiles * p.num_n_tiles;
  const int t_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * num_tiles / gridDim.x);
  const int t_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * num_tiles / gridDim.x);
  const int num_kb = (p.K + kBK - 1) / kBK;
  const int bn = p.bn;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t stage_bytes = static_cast<uint32_t>(kAStageBytes + bn * kBK * 2);
      const int box_rows = bn <= 256 ? bn : bn / 2;
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t) {
        const int m0 = (t / p.num_n_tiles) * kBM;
        const int n0 = (t % p.num_n_tiles) * bn;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], stage_bytes);
          tma_load_2d(sA + s * kAStageBytes, &tm_x, &full[s], kb * kBK, m0);
          uint8_t* b_dst = sB + s * kBStage;
          tma_load_2d(b_dst, &tm_w, &full[s], kb * kBK, n0);
          if (bn > 256) tma_load_2d(b_dst + box_rows * kBK * 2, &tm_w, &full[s], kb * kBK, n0 + box_rows);
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
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) break;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        // Gave up: wait (bounded) for the copies still in flight before the CTA's smem goes away.
        // The last min(issued, STAGES) loads sit on distinct stages, just behind stage s.
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
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const int n_sub = bn > 256 ? 2 : 1;
      const int n_mma = bn / n_sub;
      const uint32_t idesc = make_idesc_bf16(kBM, n_mma);
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t) {
        if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * MAX_BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(sA + s * kAStageBytes);
          const uint32_t b_addr = smem_u32(sB + s * kBStage);
#pragma unroll
          for (int k = 0; k < kBK / kMmaK; ++k) {
            const uint64_t a_desc = make_sdesc_sw128(a_addr + k * kMmaK * 2);
            for (int j = 0; j < n_sub; ++j) {
              const uint64_t b_desc = make_sdesc_sw128(b_addr + j * n_mma * kBK * 2 + k * kMmaK * 2);
              tc_mma_bf16(d_tmem + j * n_mma, a_desc, b_desc, idesc, (kb | k) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&empty[s]);  // frees the stage once these MMAs have read it
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);  // accumulator of this tile is complete
        if (kAccBufs == 2) {
          acc ^= 1;
          if (acc == 0) acc_ph ^= 1u;
        } else {
          acc_ph ^= 1u;
        }
      }
      if (!ok) {
        // Let every MMA issued so far finish before tensor memory is released.
        tc_commit(drain);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp < kSsFirst) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;                    // TMEM lane quarter this warp may read
    const int half = (warp - kEpiFirst) >> 2;  // which of the two warps on this quarter
    const int row_in_tile = q * 32 + lane;
    if (EPI == EPI_POSTNORM) {
      for (int i = threadIdx.x - 32 * kEpiFirst; i < p.head_dim; i += 32 * kEpiWarps) {
        const uint32_t b = p.g2[i];
        g2s[i] = __uint_as_float(b << 16);
      }
      named_bar_sync(1, 32 * kEpiWarps);
    }
    int acc = 0;
    uint32_t acc_ph = 0;
    int sb = 0;
    uint32_t sb_ph = 0;
    for (int t = t_begin; t < t_end; ++t) {
      const int mt = t / p.num_n_tiles;
      const int nt = t % p.num_n_tiles;
      if (!mbar_wait(&acc_full[acc], acc_ph, abort_flag)) break;
      tc_fence_after_sync();
      float r = 1.0f;
      if (SCALE) {
        // The explicit join: the scale of this tile's rows must be ready too.
        if (!mbar_wait(&ss_full[sb], sb_ph, abort_flag)) break;
        r = rinv[sb * kBM + row_in_tile];
        mbar_arrive(&ss_empty[sb]);
        sb ^= 1;
        if (sb == 0) sb_ph ^= 1u;
      }
      const int row = mt * kBM + row_in_tile;
      const bool row_ok = row < p.M;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * MAX_BN);

      if (EPI == EPI_LINEAR) {
        // this warp's 16-column chunks: every other one, two per TMEM wait
        const int col0 = nt * bn;
        for (int c = half * 16; c < bn; c += 64) {
          const bool two = c + 32 < bn;
          uint32_t v0[16], v1[16];
          tmem_ld16(t_row + c, v0);
          if (two) tmem_ld16(t_row + c + 32, v1);
          tmem_ld_wait();
          reg_fence16(v0);
          float o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = __uint_as_float(v0[j]) * r;
          if (row_ok) store16<OUT_F32>(p.y, p.ldy, row, col0 + c, p.n_out, o);
          if (two) {
            reg_fence16(v1);
#pragma unroll
            for (int j = 0; j < 16; ++j) o[j] = __uint_as_float(v1[j]) * r;
            if (row_ok) store16<OUT_F32>(p.y, p.ldy, row, col0 + c + 32, p.n_out, o);
          }
        }
      } else if (EPI == EPI_GLU) {
        // this warp's (gate, up) pairs of 16 columns: every other pair
        const int col0 = nt * (bn / 2);
        for (int c = half * 32; c < bn; c += 64) {
          uint32_t gt[16], up[16];
          tmem_ld16(t_row + c, gt);
          tmem_ld16(t_row + c + 16, up);
          tmem_ld_wait();
          reg_fence16(gt);
          reg_fence16(up);
          float o[16];
          const GluRow k = glu_row(r);
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = swiglu_deferred(__uint_as_float(gt[j]), __uint_as_float(up[j]), k);
          if (row_ok) store16<OUT_F32>(p.y, p.ldy, row, col0 + c / 2, p.n_out, o);
        }
      } else {  // EPI_POSTNORM
        const int hd = p.head_dim;
        const int col0 = nt * bn;
        // This row's RoPE position: >= 0 valid, -1 no RoPE, -2 outside the table (recorded in the device
        // status word; the row's rotated heads are written as NaN rather than read out of bounds).
        int rope_pos = -1;
        if (p.rope_cs != nullptr && row_ok) {
          const int ps = p.positions[row];
          if (ps >= 0 && ps < p.max_pos) {
            rope_pos = ps;
          } else {
            rope_pos = -2;
            atomicOr(&g_device_status, kStatusBadPosition);
          }
        }
        for (int h0 = 0; h0 < bn; h0 += hd) {
          // RoPE on a query/key head: rotate pairs (2i, 2i+1) by this row's (cos, sin) of pair i. The table
          // reads run one 16-column chunk ahead of their use (the first ones during the sum of squares),
          // so the epilogue does not wait on each of them.
          const bool rope_head = rope_pos >= 0 && (col0 + h0) / hd < p.n_rope_heads;
          const bool rope_bad = rope_pos == -2 && (col0 + h0) / hd < p.n_rope_heads;
          const float4* cs_row = reinterpret_cast<const float4*>(p.rope_cs) +
                                 (rope_head ? static_cast<size_t>(rope_pos) * (hd / 4) : 0);
          float4 wn[4];
          if (rope_head) {
#pragma unroll
            for (int k = 0; k < 4; ++k) wn[k] = __ldg(cs_row + k);
          }
          float ss = 0.0f;
          for (int c = 0; c < hd; c += 16) {
            uint32_t v[16];
            tmem_ld16(t_row + h0 + c, v);
            tmem_ld_wait();
            reg_fence16(v);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float u = __uint_as_float(v[j]);
              ss = fmaf(u, u, ss);
            }
          }
          const float r2 = 1.0f / sqrtf(ss / static_cast<float>(hd) + p.eps);
          for (int c = 0; c < hd; c += 16) {
            float4 w[4];
            if (rope_head) {
#pragma unroll
              for (int k = 0; k < 4; ++k) w[k] = wn[k];
              if (c + 16 < hd) {
#pragma unroll
                for (int k = 0; k < 4; ++k) wn[k] = __ldg(cs_row + (c + 16) / 4 + k);
              }
            }
            uint32_t v[16];
            tmem_ld16(t_row + h0 + c, v);
            tmem_ld_wait();
            reg_fence16(v);
            float o[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) o[j] = __uint_as_float(v[j]) * r2 * g2s[c + j];
            if (rope_head) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {  // w[k]: (cos, sin) of pairs c/2 + 2k and c/2 + 2k + 1
                const float a0 = o[4 * k], b0 = o[4 * k + 1], a1 = o[4 * k + 2], b1 = o[4 * k + 3];
                o[4 * k] = a0 * w[k].x - b0 * w[k].y;
                o[4 * k + 1] = a0 * w[k].y + b0 * w[k].x;
                o[4 * k + 2] = a1 * w[k].z - b1 * w[k].w;
                o[4 * k + 3] = a1 * w[k].w + b1 * w[k].z;
              }
            } else if (rope_bad) {
#pragma unroll
              for (int j = 0; j < 16; ++j) o[j] = __int_as_float(0x7FC00000);
            }
            if (row_ok) store16<OUT_F32>(p.y, p.ldy, row, col0 + h0 + c, p.n_out, o);
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (kAccBufs == 2) {
        acc ^= 1;
        if (acc == 0) acc_ph ^= 1u;
      } else {
        acc_ph ^= 1u;
      }
    }
  } else if (SCALE) {
    // ------------------------------------------------------------------ sum of squares (deferred norm)
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int s = 0;
    uint32_t ph = 0;
    int sb = 0;
    uint32_t sb_ph = 0;
    bool ok = true;
    int last_m = -1;  // row block whose 1/rms this thread holds in `r_row`
    float r_row = 0.0f;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const int mt = t / p.num_n_tiles;
      const bool fresh = mt != last_m;  // same for the whole CTA
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      for (int kb = 0; kb < num_kb; ++kb) {
        // Every stage use gets this warp's release (the stage barriers count it), and the warp waits
        // for every use's data, reading it only when the row block's sum of squares is not known yet.
        // The wait matters even when nothing is read: a parity wait tells its phase apart only from the
        // phase just before it. A warp that skipped the data waits could run ahead, release a use the
        // TMA had not filled yet, and then, on the next row block, find the full barrier's phase
        // two uses back completed (same parity), take it as this use, read stale x and arrive a
        // second time on the earlier phase of `empty`. That phase would then complete without the MMA's
        // commit, the refill would overlap a load in flight, and a later full phase would never
        // collect its bytes.
        if (!mbar_wait(&full[s], ph, abort_flag)) {
          ok = false;
          break;
        }
        // Row `row_in_tile` of the x tile is one 128-byte line (its 16-byte chunks are permuted by
        // the swizzle, which does not matter for a sum). Lanes start at different chunks so that
        // each quarter-warp covers all 32 banks.
        const uint8_t* line = sA + s * kAStageBytes + row_in_tile * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (!fresh) break;
          const uint4 w = *reinterpret_cast<const uint4*>(line + (((c ^ lane) & 7) << 4));
          float f;
          f = bf16lo_to_f32(w.x); a0 = fmaf(f, f, a0);
          f = bf16hi_to_f32(w.x); a1 = fmaf(f, f, a1);
          f = bf16lo_to_f32(w.y); a2 = fmaf(f, f, a2);
          f = bf16hi_to_f32(w.y); a3 = fmaf(f, f, a3);
          f = bf16lo_to_f32(w.z); a0 = fmaf(f, f, a0);
          f = bf16hi_to_f32(w.z); a1 = fmaf(f, f, a1);
          f = bf16lo_to_f32(w.w); a2 = fmaf(f, f, a2);
          f = bf16hi_to_f32(w.w); a3 = fmaf(f, f, a3);
        }
        // The generic-proxy reads above must be ordered before the TMA (async proxy) refill of this
        // stage that our arrival permits.
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      if (fresh) {
        const float ss = (a0 + a1) + (a2 + a3);
        r_row = 1.0f / sqrtf(ss / static_cast<float>(p.K) + p.eps);
        last_m = mt;
      }
      if (!mbar_wait(&ss_empty[sb], sb_ph ^ 1u, abort_flag)) break;
      rinv[sb * kBM + row_in_tile] = r_row;
      mbar_arrive(&ss_full[sb]);
      sb ^= 1;
      if (sb == 0) sb_ph ^= 1u;
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace fn
