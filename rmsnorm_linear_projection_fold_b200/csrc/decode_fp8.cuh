// decode_fp8.cuh — decode-sized FlashNorm projections (M <= 16 tokens) with FP8 E4M3 folded weights,
// on the tensor cores.
//
//     y[m, n] = (sum_k x[m, k] dec(Q[n, k])) * s[n] * 1/sqrt(mean_k x[m, k]^2 + eps)
//
// ("FlashNorm: Fast Normalization for Transformers", Abstract: folded weights stay compatible with
// quantized models; the gain is folded before quantization and the deferred 1/rms multiplies the output
// together with the channel's dequantization scale s[n].)
//
// The weights stream from HBM as one byte each. A tensor-core MMA needs both operands in one 16-bit
// type, so the E4M3 codes are widened on chip, exactly, to f16 (every E4M3 value is an f16), and the
// activations are given to the MMA as f16 too, scaled per token by a power of two chosen from the
// token's largest |x| (x * 2^e lies in [2^14, 2^15) at its largest), so that every bf16 activation is
// exactly an f16 (or, below 2^-29 of its token's largest element, off by less than 2^-40 of it). The
// accumulator is multiplied back by 2^-e, exactly, in the epilogue.
//
// Per CTA, one slab of 128 W* rows (the MMA's M side; the <= 16 tokens are its N side) over one range
// of K:
//   warp 0      TMA producer: 128 rows x 128 codes (16 KB) per stage, 128-byte swizzle
//   warp 1      tensor-memory allocator; one lane issues the MMAs, A read from tensor memory
//   warps 2-5   converters: each thread widens its W* row of a stage (128 codes) to f16 and writes it
//               to an A buffer in tensor memory (tcgen05.st), then runs the epilogue for that row
//   warps 6-9   activations: per token the sum of squares (the deferred norm, from the exact bf16
//               values) and the largest |x| over this CTA's K range, then x * 2^e as f16 into the
//               resident, swizzled B tile in shared memory
// The sum of squares and the contraction run at the same time on different warps and meet in the
// epilogue, the explicit join of the other kernels. When there are few slabs, K is split across a
// cluster of `ksplit` CTAs and the partial accumulators and sums of squares are added in the leader
// CTA through distributed shared memory, in a fixed order.
#pragma once

#include "sm100.cuh"

namespace fn {

constexpr int kD8Rows = 128;                  // W* rows per CTA (MMA M)
constexpr int kD8Tok = 16;                    // token slots (MMA N)
constexpr int kD8KStage = 128;                // k per stage: 128 one-byte codes, one 128-byte row
constexpr int kD8WStage = kD8Rows * kD8KStage;  // 16 KB
constexpr int kD8Stages = 3;
constexpr int kD8ABufs = 3;                   // f16 A tiles in tensor memory, 64 columns each
constexpr int kD8ACol0 = 64;                  // first A column (the accumulator takes columns 0..15)
constexpr int kD8Threads = 320;
constexpr int kD8XUnit = kD8Tok * kD8KStage * 2;  // B tile bytes per stage unit: 16 tokens x 128 k, f16

struct DecodeFp8Params {
  void* y;
  const uint16_t* x;     // bf16 [M, K]
  const float* scales;   // fp32 [N]
  int M, K, N, ldy;
  int ksplit;
  float eps;
};

// Dynamic shared memory for a CTA whose K range spans at most `units` stages of 128.
__host__ __device__ constexpr int decode_fp8_smem_bytes(int units, int ksplit) {
  return 1024 + kD8Stages * kD8WStage + units * kD8XUnit +
         (ksplit > 1 ? (ksplit - 1) * kD8Rows * kD8Tok * 4 + ksplit * kD8Tok * 4 : 0) + 512;
}

// Instruction descriptor for kind::f16 with f16 A and B, fp32 D, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t make_idesc_f16(int m, int n) {
  return (1u << 4)                                  // D format: f32 (A, B format 0: f16)
         | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24);   // M / 16
}

// D[tmem] (+)= A[tmem] * B[smem]^T, f16 inputs, fp32 accumulate; A is read from tensor memory.
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Store 32 consecutive 32-bit tensor-memory columns of this thread's lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Two E4M3 codes (bits 0-7 and 8-15 of `c`) to f16x2, exactly: code 0-7 to the low half.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t c) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(c));
  return r;
}

// Two floats to f16x2 (round to nearest even); `lo` goes to the lower address.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int KSPLIT, bool OUT_F32>
__global__ void __launch_bounds__(kD8Threads, 2)
    k_decode_fp8(const __grid_constant__ CUtensorMap tm_q, DecodeFp8Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const int num_units = (p.K + kD8KStage - 1) / kD8KStage;          // stages of 128 over all of K
  const int max_units = (num_units + KSPLIT - 1) / KSPLIT;          // the longest K range of a CTA
  uint8_t* sW = smem;                                               // [kD8Stages][128 rows][128 codes]
  uint8_t* sX = sW + kD8Stages * kD8WStage;                         // [units][2 atoms][16 rows x 128 B]
  float* part_d = reinterpret_cast<float*>(sX + max_units * kD8XUnit);  // [KSPLIT-1][128][16] (leader)
  float* part_ss = part_d + (KSPLIT > 1 ? (KSPLIT - 1) * kD8Rows * kD8Tok : 0);  // [KSPLIT][16]
  uint64_t* full = reinterpret_cast<uint64_t*>(part_ss + (KSPLIT > 1 ? KSPLIT * kD8Tok : 0));
  uint64_t* empty = full + kD8Stages;
  uint64_t* afull = empty + kD8Stages;
  uint64_t* aempty = afull + kD8ABufs;
  uint64_t* xready = aempty + kD8ABufs;
  uint64_t* acc_full = xready + 1;
  uint64_t* drain = acc_full + 1;
  float* tok_ss = reinterpret_cast<float*>(drain + 1);   // [16] this CTA's sum of squares per token
  float* tok_sc = tok_ss + kD8Tok;                        // [16] 2^-e per token
  float* rs = tok_sc + kD8Tok;                            // [16] 1/rms per token (leader)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rs + kD8Tok);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) >> 5, 0);
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const uint32_t rank = KSPLIT > 1 ? cluster_ctarank() : 0;
  const int slab = static_cast<int>(blockIdx.x) / KSPLIT;
  const int n0 = slab * kD8Rows;
  const int u0 = static_cast<int>((static_cast<long long>(rank) * num_units) / KSPLIT);
  const int u1 = static_cast<int>((static_cast<long long>(rank + 1) * num_units) / KSPLIT);
  const int k_lo = u0 * kD8KStage;
  const int k_hi = min(u1 * kD8KStage, p.K);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kD8Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);  // the four converter warps
    }
    for (int b = 0; b < kD8ABufs; ++b) {
      mbar_init(&afull[b], 4);  // the four converter warps
      mbar_init(&aempty[b], 1);  // the MMA's commit
    }
    mbar_init(xready, 4);  // the four activation warps
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tm_q);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();  // the previous kernel's outputs (our inputs, or buffers we overwrite) are complete

  const float kNaN = __int_as_float(0x7fc00000);
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int u = u0; u < u1; ++u) {
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], kD8WStage);
        tma_load_2d(sW + s * kD8WStage, &tm_q, &full[s], u * kD8KStage, n0);
        ++issued;
        if (++s == kD8Stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      grid_dep_launch();  // all loads issued: the next kernel may be scheduled onto SMs as they free up
      if (!ok) {
        const int pending = issued < kD8Stages ? issued : kD8Stages;
        for (int i = 1; i <= pending; ++i) {
          int st = s - i;
          uint32_t pp = ph;
          if (st < 0) {
            st += kD8Stages;
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
      const uint32_t idesc = make_idesc_f16(kD8Rows, kD8Tok);
      int b = 0;
      uint32_t ph = 0;
      bool ok = mbar_wait(xready, 0, abort_flag);
      for (int u = u0; u < u1 && ok; ++u) {
        if (!mbar_wait(&afull[b], ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_col = tmem_base + static_cast<uint32_t>(kD8ACol0 + b * 64);
        const uint32_t x_unit = smem_u32(sX + (u - u0) * kD8XUnit);
#pragma unroll
        for (int j = 0; j < kD8KStage / 16; ++j)  // 8 MMAs of K = 16: 8 columns of A, 32 bytes of a B row
          tc_mma_f16_ts(tmem_base, a_col + j * 8, make_sdesc_sw128(x_unit + (j >> 2) * 2048 + (j & 3) * 32), idesc,
                        (u != u0 || j != 0) ? 1u : 0u);
        tc_commit(&aempty[b]);  // the A buffer may be refilled once these MMAs have read it
        if (++b == kD8ABufs) {
          b = 0;
          ph ^= 1u;
        }
      }
      tc_commit(ok ? acc_full : drain);
      if (ok) {
        // wait for every A buffer's last release: no commit arrival is still in flight at exit
        const int n = u1 - u0;
        for (int j = 0; j < kD8ABufs; ++j) {
          const int uses = (n - j + kD8ABufs - 1) / kD8ABufs;
          if (uses > 0 && !mbar_wait(&aempty[j], static_cast<uint32_t>(uses - 1) & 1u, abort_flag)) break;
        }
      } else {
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------------ activations (warps 6-9)
    // 8 threads per token; each takes every 8th 16-byte chunk (8 values) of the token's K range.
    const int t = static_cast<int>(threadIdx.x) - 192;  // 0..127
    const int tok = t >> 3, sub = t & 7;
    float ss = 0.f, mx = 0.f;
    const bool live = tok < p.M;
    const uint16_t* xr = p.x + static_cast<size_t>(tok) * p.K;
    if (live) {
      for (int k = k_lo + sub * 8; k < k_hi; k += 64) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(xr + k));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float a = bf16lo_to_f32(ws[i]), b = bf16hi_to_f32(ws[i]);
          ss = fmaf(a, a, ss);
          ss = fmaf(b, b, ss);
          mx = fmaxf(mx, fmaxf(fabsf(a), fabsf(b)));
        }
      }
    }
#pragma unroll
    for (int o = 4; o >= 1; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    // x * 2^e with the largest |x| in [2^14, 2^15): every bf16 value of the token at most 29 binades
    // below the largest is then an f16 normal and converts exactly.
    int ex = 0;
    if (mx > 0.f) {
      int e2;
      frexpf(mx, &e2);  // mx = f * 2^e2, f in [0.5, 1)
      ex = min(max(15 - e2, -120), 120);
    }
    const float up = ldexpf(1.0f, ex);
    if (sub == 0) {
      tok_ss[tok] = ss;
      tok_sc[tok] = ldexpf(1.0f, -ex);
    }
    // the B tile: unit v = (k - k_lo) / 128, atom a = 64-k half, row = token, 16-byte chunk c of the
    // 128-byte row at c ^ (row & 7) (the 128-byte swizzle the MMA descriptor expects)
    for (int k = k_lo + sub * 8; k < k_lo + (u1 - u0) * kD8KStage; k += 64) {
      uint4 o = make_uint4(0u, 0u, 0u, 0u);
      if (live && k < k_hi) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(xr + k));
        o.x = pack_f16x2(bf16lo_to_f32(w.x) * up, bf16hi_to_f32(w.x) * up);
        o.y = pack_f16x2(bf16lo_to_f32(w.y) * up, bf16hi_to_f32(w.y) * up);
        o.z = pack_f16x2(bf16lo_to_f32(w.z) * up, bf16hi_to_f32(w.z) * up);
        o.w = pack_f16x2(bf16lo_to_f32(w.w) * up, bf16hi_to_f32(w.w) * up);
      }
      const int kk = k - k_lo;
      const int v = kk / kD8KStage, a = (kk % kD8KStage) / 64, c = (kk % 64) / 8;
      uint8_t* dst = sX + v * kD8XUnit + a * 2048 + (tok >> 3) * 1024 + (tok & 7) * 128 + ((c ^ (tok & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = o;
    }
    fence_proxy_async_smem();  // generic stores above, read by the MMA (async proxy)
    __syncwarp();
    if (lane == 0) mbar_arrive(xready);
  } else {
    // ------------------------------------------------------------------ converters (warps 2-5), epilogue
    const int q = warp & 3;                 // tensor-memory lane quarter
    const int row = q * 32 + lane;          // W* row within the slab
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int s = 0, b = 0;
    uint32_t ph = 0, bph = 0;
    bool ok = true;
    for (int u = u0; u < u1; ++u) {
      if (!mbar_wait(&full[s], ph, abort_flag) || !mbar_wait(&aempty[b], bph ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      // this row's 128 codes: eight 16-byte chunks, chunk c at c ^ (row & 7) (TMA's 128-byte swizzle)
      const uint8_t* line = sW + s * kD8WStage + row * 128;
      uint32_t h[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = half * 4 + c4;
          const uint4 w = *reinterpret_cast<const uint4*>(line + (((c ^ row) & 7) << 4));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            h[c4 * 8 + 2 * i] = e4m3x2_to_f16x2(ws[i] & 0xFFFFu);
            h[c4 * 8 + 2 * i + 1] = e4m3x2_to_f16x2(ws[i] >> 16);
          }
        }
        tmem_st32(tmem_base + lane_base + static_cast<uint32_t>(kD8ACol0 + b * 64 + half * 32), h);
      }
      fence_proxy_async_smem();  // the reads above come before the TMA refill this arrival permits
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[s]);
        mbar_arrive(&afull[b]);
      }
      if (++s == kD8Stages) {
        s = 0;
        ph ^= 1u;
      }
      if (++b == kD8ABufs) {
        b = 0;
        bph ^= 1u;
      }
    }
    // the accumulator of this row: 16 tokens, scaled back by 2^-e per token
    float v[kD8Tok];
    if (ok) ok = mbar_wait(acc_full, 0, abort_flag) && mbar_wait(xready, 0, abort_flag);
    if (ok && u1 > u0) {
      tc_fence_after_sync();
      uint32_t r[16];
      tmem_ld16(tmem_base + lane_base, r);
      tmem_ld_wait();
      reg_fence16(r);
#pragma unroll
      for (int j = 0; j < kD8Tok; ++j) v[j] = __uint_as_float(r[j]) * tok_sc[j];
    } else {
      // an empty K range contributes zero; a wait that gave up contributes NaN
#pragma unroll
      for (int j = 0; j < kD8Tok; ++j) v[j] = ok ? 0.f : kNaN;
    }
    const int t = static_cast<int>(threadIdx.x) - 64;  // 0..127
    float ss_part = 0.f;
    if (t < kD8Tok) ss_part = ok ? tok_ss[t] : kNaN;
    if (KSPLIT > 1 && rank != 0) {
      const uint32_t dst = dsmem_addr(part_d + ((rank - 1) * kD8Rows + row) * kD8Tok, 0);
#pragma unroll
      for (int j = 0; j < kD8Tok; j += 4) dsmem_st_v4(dst + j * 4, v[j], v[j + 1], v[j + 2], v[j + 3]);
      if (t < kD8Tok) dsmem_st_f32(dsmem_addr(part_ss + rank * kD8Tok + t, 0), ss_part);
    }
    if (KSPLIT > 1) cluster_sync_all();  // the partial sums have reached the leader
    if (rank == 0) {
      if (KSPLIT > 1) {
        for (int rr = 1; rr < KSPLIT; ++rr) {
#pragma unroll
          for (int j = 0; j < kD8Tok; ++j) v[j] += part_d[((rr - 1) * kD8Rows + row) * kD8Tok + j];
          if (t < kD8Tok) ss_part += part_ss[rr * kD8Tok + t];
        }
      }
      if (t < kD8Tok) rs[t] = 1.0f / sqrtf(ss_part / static_cast<float>(p.K) + p.eps);
      named_bar_sync(1, 128);
      const int n = n0 + row;
      if (n < p.N) {
        const float sc = p.scales[n];
#pragma unroll
        for (int m = 0; m < kD8Tok; ++m) {
          if (m >= p.M) break;
          const float o = v[m] * sc * rs[m];
          if (OUT_F32)
            static_cast<float*>(p.y)[static_cast<size_t>(m) * p.ldy + n] = o;
          else
            static_cast<uint16_t*>(p.y)[static_cast<size_t>(m) * p.ldy + n] =
                static_cast<uint16_t>(pack_bf16x2(o, 0.f) & 0xFFFFu);
        }
      }
    }
  }
  if (KSPLIT > 1 && (warp < 2 || warp >= 6)) cluster_sync_all();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, 256);
}

}  // namespace fn
