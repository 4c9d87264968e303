// decode_fp8.cuh — decode-sized FlashNorm projections (M <= 16 tokens) with FP8 E4M3 folded weights,
// on the tensor cores.
//
//     y[m, n] = (sum_k x[m, k] dec(Q[n, k])) * s[n] * 1/sqrt(mean_k x[m, k]^2 + eps)
//
// ("FlashNorm: Fast Normalization for Transformers", Abstract: folded weights stay compatible with
// quantized models; the gain is folded before quantization and the deferred 1/rms multiplies the output
// together with the channel's dequantization scale s[n].)
//
// The weights stream from HBM as one byte each. A tensor-core MMA of kind::f16 takes both operands in
// one 16-bit type, so the E4M3 codes are widened on chip, exactly, to bf16 (every E4M3 value is a bf16)
// and the activations go to the MMA as they are. The widening is integer arithmetic plus one packed
// bf16 multiply per two codes (e4m3_pairs_to_bf16x2), not the hardware E4M3 conversion, whose
// throughput is a fraction of the rate HBM delivers codes at. The widened tile is written straight into
// tensor memory, and the MMA reads its A operand from there: the codes cross shared memory once (TMA
// in, the converters out), not three times.
//
// Per CTA, one slab of 128 W* rows (the MMA's M side; the <= 16 tokens are its N side) over one range
// of K, in stages of 128 k (128 codes per W* row, 16 KB, and 16 x 128 bf16 of x, 4 KB):
//   warp 0      TMA producer
//   warp 1      tensor-memory allocator; lane 0 issues the MMAs of every kD8Issuers-th stage (A from
//               tensor memory, B = the x tile); warps 6.. issue the others'
//   warps 2-5   converters: each thread widens its W* row of a stage to bf16 into an A buffer in tensor
//               memory (tcgen05.st) and adds up x^2 for one token over 16 of the stage's k (the
//               deferred norm, from the same staged x tiles the MMA reads); then the epilogue
// A stage is refilled once the converters have read it and the MMA that read its x tile has completed.
// When there are few slabs, K is split in `ksplit` ranges, one CTA each. Either the CTAs of a slab form a
// cluster and the partial accumulators and sums of squares are added in the leader CTA through
// distributed shared memory (KSPLIT > 1), or (KSPLIT == 0, a caller workspace) they are independent CTAs
// that write their partials to the workspace and count their arrivals on the slab's counter: the CTA
// that arrives last adds the partials in K order and writes the output. Nothing waits on another CTA,
// the sum is in a fixed order whichever CTA comes last, and the ranges need no co-scheduling, so two
// 5-stage CTAs can share every SM.
#pragma once

#include "sm100.cuh"

namespace fn {

constexpr int kD8Rows = 128;                       // W* rows per CTA (MMA M)
constexpr int kD8Tok = 16;                         // token slots (MMA N)
constexpr int kD8KStage = 128;                     // k per stage: 128 one-byte codes, one 128-byte row
constexpr int kD8WStage = kD8Rows * kD8KStage;     // 16 KB of codes
constexpr int kD8XStage = kD8Tok * kD8KStage * 2;  // 4 KB of x: two 64-k atoms of 16 rows x 128 bytes
// Formats of the quantized W*. FP8 E4M3: one byte per weight; a pipeline stage is one 128-k unit (a
// 128-byte row per W* row, 128-byte swizzle). NVFP4: E2M1 codes with E4M3 scales per 16 k, stored in
// groups of 256 k of 144 bytes per W* row (fp8.cuh); a stage is one group, two 128-k units, loaded
// without swizzle: rows 144 bytes apart put the eight rows of a quarter warp on distinct banks.
constexpr int kFmtFp8 = 0, kFmtNvfp4 = 1;
template <int FMT>
struct D8Fmt {
  static constexpr int kUnits = FMT == kFmtNvfp4 ? 2 : 1;         // 128-k units per stage
  static constexpr int kRowBytes = FMT == kFmtNvfp4 ? 144 : 128;  // bytes of one W* row per stage
  static constexpr int kWStage = kD8Rows * kRowBytes;
  static constexpr int kXStage = kUnits * kD8XStage;
  static constexpr int kKStage = kUnits * kD8KStage;  // k per stage
};
constexpr int kD8ABufs = 3;                        // bf16 A tiles in tensor memory, 64 columns each
constexpr int kD8ACol0 = 64;                       // first A column (the accumulators take columns 0..63)
// MMA issuers: stage i of a CTA's K range is issued by issuer i % kD8Issuers, into that issuer's own
// kD8Accs / kD8Issuers accumulators (MMA j of the stage into the issuer's accumulator j % that count);
// the epilogue adds the kD8Accs accumulators in a fixed order. One thread issuing back-to-back
// M = 128, N = 16 MMAs gets one through every ~60 cycles, and every ~125 while other warps store to
// tensor memory (the converters do): per-issuer cost, not tensor-core throughput, so issuers in
// separate warps overlap almost linearly.
constexpr int kD8Accs = 4;
constexpr int kD8Issuers = 2;
constexpr int kD8AccPer = kD8Accs / kD8Issuers;
static_assert(kD8Accs % kD8Issuers == 0, "each issuer owns the same number of accumulators");
// The issuer of stage i + kD8ABufs (which reuses stage i's A buffer) last waited on stage
// i + kD8ABufs - kD8Issuers; that must not come before stage i, or its parity wait on the buffer's
// barrier could see stage i's phase, one phase early. Likewise for the stage ring (at least 4 stages).
static_assert(kD8Issuers <= kD8ABufs && kD8Issuers <= 4, "an issuer would run a barrier phase ahead");
// warp 0 TMA, warp 1 allocator + issuer 0, warps 2-5 converters, warps 6.. issuers 1..
constexpr int kD8Threads = 192 + 32 * (kD8Issuers - 1);
// Workspace of the KSPLIT == 0 kernel: kD8MaxWsSlabs arrival counters (uint32), then the partials
// [slab][range][128 rows][16 tokens] fp32, then the partial sums of squares [slab][range][16] fp32.
constexpr int kD8MaxWsSlabs = 256;
constexpr int kD8WsCounterBytes = kD8MaxWsSlabs * 4;

struct DecodeFp8Params {
  void* y;
  const float* scales;  // fp32 [N]
  int M, K, N, ldy;
  int ksplit;
  float eps;
  unsigned* counters;  // KSPLIT == 0: one per slab, zero between calls
  float* part;         // KSPLIT == 0: [slabs][ksplit][128][16]
  float* part_ss;      // KSPLIT == 0: [slabs][ksplit][16]
};

template <int STAGES, int KSPLIT, int FMT = kFmtFp8>
__host__ __device__ constexpr int decode_fp8_smem_bytes() {
  return 1024 + STAGES * (D8Fmt<FMT>::kWStage + D8Fmt<FMT>::kXStage) +
         (KSPLIT > 1 ? (KSPLIT - 1) * kD8Rows * kD8Tok * 4 + KSPLIT * kD8Tok * 4 : 0) + 512;
}

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 inputs, fp32 accumulate; A is read from tensor memory.
__device__ __forceinline__ void tc_mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
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

// Two E4M3 codes, one in the low byte of each 16-bit half of `v` (the high bytes zero), to bf16x2,
// exactly. Shifted left by 4, a code s.eeee.mmm (bias 7) has eeee at bits 10-7 and mmm at bits 6-4, the
// places of a bf16's low exponent bits and top mantissa bits, and its sign at bit 11; adding 15 times
// that sign bit moves it to bit 15 (0x0800 + 0x7800 = 0x8000). The bf16 read from those bits is
// 2^(e-127) (1 + m/8) (for e = 0 the bf16 subnormal m/8 2^-126); one multiply by 2^120 makes it the
// E4M3 value 2^(e-7) (1 + m/8) (or m 2^-9), exact in bf16, zero and -0 included.
__device__ __forceinline__ uint32_t e4m3_pairs_to_bf16x2(uint32_t v) {
  const uint32_t t = v << 4;
  const uint32_t f = (t & 0x08000800u) * 15u + t;
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(f), "r"(0x7B807B80u));  // x 2^120
  return r;
}

// Two E2M1 codes, the even k in bits 0..3 of `v` and the odd k in bits 16..19, to bf16x2 weights times
// 2^-63, exactly. A code s.ee.m has ee at bits 2..1 and m at bit 0; moved to bits 8..7 and 6 (a bf16's low
// exponent bits and top mantissa bit), with s at bit 15, the bf16 read from those bits is 2^(ee-127)(1 +
// m/2) (for ee = 0 the subnormal m 2^-127): 2^-126 times the E2M1 value 2^(ee-1)(1 + m/2) (or m/2). One
// multiply by scale2 = the block scale times 2^63 makes it the weight times 2^-63: at most 6 significant
// bits (E2M1's 2, E4M3's 4) and, for block scales of 2^-9 .. 448, magnitudes of 2^-73 .. 2^-52, normal in
// bf16, so the product is exact. The epilogue multiplies the accumulator by 2^63 (kNvfp4Unscale).
__device__ __forceinline__ uint32_t e2m1_pair_to_bf16x2(uint32_t v, uint32_t scale2) {
  const uint32_t f = ((v & 0x00070007u) << 6) | ((v & 0x00080008u) << 12);
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(f), "r"(scale2));
  return r;
}
constexpr float kNvfp4Unscale = 9223372036854775808.0f;  // 2^63

template <int STAGES, int KSPLIT, bool OUT_F32, int FMT = kFmtFp8>
__global__ void __launch_bounds__(kD8Threads, 1)
    k_decode_fp8(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_x,
                 DecodeFp8Params p) {
  using F = D8Fmt<FMT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sW = smem;                       // [STAGES][128 rows][F::kRowBytes]
  uint8_t* sX = sW + STAGES * F::kWStage;   // [STAGES][2 atoms per unit][16 rows x 128 bytes], 128-byte swizzle
  float* part_d = reinterpret_cast<float*>(sX + STAGES * F::kXStage);            // [KSPLIT-1][128][16]
  float* part_ss = part_d + (KSPLIT > 1 ? (KSPLIT - 1) * kD8Rows * kD8Tok : 0);  // [KSPLIT][16]
  uint64_t* full = reinterpret_cast<uint64_t*>(part_ss + (KSPLIT > 1 ? KSPLIT * kD8Tok : 0));
  uint64_t* empty = full + STAGES;
  uint64_t* afull = empty + STAGES;
  uint64_t* aempty = afull + kD8ABufs;
  uint64_t* acc_full = aempty + kD8ABufs;
  uint64_t* drain = acc_full + 1;                             // [kD8Issuers]
  float* rs = reinterpret_cast<float*>(drain + kD8Issuers);  // [16] 1/rms per token (leader)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rs + kD8Tok);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;  // KSPLIT == 0: this CTA arrived last on its slab

  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) >> 5, 0);
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const int ks = KSPLIT == 0 ? p.ksplit : KSPLIT;  // K ranges per slab
  const uint32_t rank = KSPLIT == 0 ? blockIdx.x % static_cast<uint32_t>(ks) : (KSPLIT > 1 ? cluster_ctarank() : 0);
  const int slab = static_cast<int>(blockIdx.x) / ks;
  const int n0 = slab * kD8Rows;
  // this range's 128-k units [u0, u1), split evenly over the ranges; it loads the stages [g0, g1) that
  // hold them (with NVFP4 a range may start or end in the middle of a 256-k stage)
  const int num_units = (p.K + F::kKStage - 1) / F::kKStage * F::kUnits;
  const int u0 = static_cast<int>((static_cast<long long>(rank) * num_units) / ks);
  const int u1 = static_cast<int>((static_cast<long long>(rank + 1) * num_units) / ks);
  const int g0 = u0 / F::kUnits, g1 = u1 > u0 ? (u1 + F::kUnits - 1) / F::kUnits : g0;  // an empty range loads nothing

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4 + F::kUnits);  // the four converter warps and the commit of each unit's MMAs
    }
    for (int b = 0; b < kD8ABufs; ++b) {
      mbar_init(&afull[b], 4);   // the four converter warps
      mbar_init(&aempty[b], 1);  // the MMA's commit
    }
    mbar_init(acc_full, kD8Issuers);  // each issuer's last commit
    for (int i = 0; i < kD8Issuers; ++i) mbar_init(&drain[i], 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_x);
    // the first ring's worth of this CTA's codes into L2 while the previous kernel drains
    for (int gi = g0; gi < g1 && gi < g0 + STAGES; ++gi) tma_prefetch_l2_2d(&tm_q, gi * F::kRowBytes, n0);
  }
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
      for (int gi = g0; gi < g1; ++gi) {
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], F::kWStage + F::kXStage);
        tma_load_2d(sW + s * F::kWStage, &tm_q, &full[s], gi * F::kRowBytes, n0);
#pragma unroll
        for (int a = 0; a < 2 * F::kUnits; ++a)  // x in 64-k atoms
          tma_load_2d(sX + s * F::kXStage + a * 2048, &tm_x, &full[s], gi * F::kKStage + 64 * a, 0);
        ++issued;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      grid_dep_launch();  // all loads issued: the next kernel may be scheduled onto SMs as they free up
      if (ok) {
        // wait for every stage's last release: no MMA commit arrival is in flight at exit
        for (int i = 0; i < STAGES; ++i) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) break;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      } else {
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
  } else if (warp == 1 || warp >= 6) {
    // ------------------------------------------------------------------ MMA issuers
    const int iss = warp == 1 ? 0 : warp - 5;  // stages iss, iss + kD8Issuers, ... of this CTA's range
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(kD8Rows, kD8Tok);
      const uint32_t acc0 = tmem_base + static_cast<uint32_t>(iss * kD8AccPer * kD8Tok);
      bool ok = true;
      for (int i = iss; u0 + i < u1; i += kD8Issuers) {  // unit i of the range
        const int u = u0 + i, st = u / F::kUnits - g0;   // its stage, counted from the range's first
        const int s = st % STAGES, b = i % kD8ABufs;
        const uint32_t ph = static_cast<uint32_t>(st / STAGES) & 1u, bph = static_cast<uint32_t>(i / kD8ABufs) & 1u;
        // the x tile of this stage (TMA) and the widened codes in A buffer b (the converters)
        if (!mbar_wait(&full[s], ph, abort_flag) || !mbar_wait(&afull[b], bph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_col = tmem_base + static_cast<uint32_t>(kD8ACol0 + b * 64);
        const uint32_t x_st = smem_u32(sX + s * F::kXStage + (u % F::kUnits) * kD8XStage);
#pragma unroll
        for (int j = 0; j < kD8KStage / 16; ++j)  // 8 MMAs of K = 16: 8 columns of A, 32 bytes of a B row
          tc_mma_bf16_ts(acc0 + static_cast<uint32_t>((j % kD8AccPer) * kD8Tok), a_col + j * 8,
                         make_sdesc_sw128(x_st + (j >> 2) * 2048 + (j & 3) * 32), idesc,
                         (i != iss || j >= kD8AccPer) ? 1u : 0u);
        tc_commit(&aempty[b]);  // A buffer b may be refilled once these MMAs have read it
        tc_commit(&empty[s]);   // and the stage, whose x tile they read
      }
      tc_commit(ok ? acc_full : &drain[iss]);
      if (!ok) {
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(&drain[iss], 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ converters (warps 2-5), epilogue
    const int q = warp & 3;                 // tensor-memory lane quarter
    const int row = q * 32 + lane;          // W* row within the slab
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int t = static_cast<int>(threadIdx.x) - 64;  // 0..127
    const int tok = t >> 3, sub = t & 7;    // sum of squares: token, and its 16-byte chunk of each atom row
    bool ok = true;
    float ss = 0.f;
    // this row's dequantization scale, loaded now so that its latency hides under the main loop
    const float sc = n0 + row < p.N ? p.scales[n0 + row] : 0.f;
    for (int i = 0; u0 + i < u1; ++i) {  // unit i of the range: half `half` of its stage
      const int u = u0 + i, st = u / F::kUnits - g0, half = u % F::kUnits;
      const int s = st % STAGES, b = i % kD8ABufs;
      const uint32_t ph = static_cast<uint32_t>(st / STAGES) & 1u, bph = static_cast<uint32_t>(i / kD8ABufs) & 1u;
      if (!mbar_wait(&full[s], ph, abort_flag) || !mbar_wait(&aempty[b], bph ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t a_st = tmem_base + lane_base + static_cast<uint32_t>(kD8ACol0 + b * 64);
      if constexpr (FMT == kFmtFp8) {
        // this row's 128 codes: eight 16-byte chunks, chunk c at c ^ (row & 7) (TMA's 128-byte swizzle)
        const uint8_t* line = sW + s * F::kWStage + row * 128;
        uint32_t h[32];
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c = q2 * 4 + c4;
            const uint4 w = *reinterpret_cast<const uint4*>(line + (((c ^ row) & 7) << 4));
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {  // codes k0..k3 of word e: columns (k0, k1) and (k2, k3)
              h[c4 * 8 + 2 * e] = e4m3_pairs_to_bf16x2(__byte_perm(ws[e], 0u, 0x4140));
              h[c4 * 8 + 2 * e + 1] = e4m3_pairs_to_bf16x2(__byte_perm(ws[e], 0u, 0x4342));
            }
          }
          tmem_st32(a_st + static_cast<uint32_t>(q2 * 32), h);
        }
      } else {
        // this row's group of 144 bytes: unit `half` is code words 16 half .. + 15 (blocks 8 half .. + 7,
        // two words each) and block scales 128 + 8 half .. + 7
        const uint8_t* line = sW + s * F::kWStage + row * 144;
        const uint2 scw = *reinterpret_cast<const uint2*>(line + 128 + 8 * half);
        uint32_t h[32];
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {  // 32 columns: blocks 4 q2 .. 4 q2 + 3
#pragma unroll
          for (int c = 0; c < 2; ++c) {  // one 16-byte chunk: two blocks
            const uint4 w = *reinterpret_cast<const uint4*>(line + (half * 4 + q2 * 2 + c) * 16);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int bb = q2 * 4 + c * 2 + e;  // block of this unit: columns 8 bb .. 8 bb + 7
              const uint32_t sbyte = ((bb < 4 ? scw.x : scw.y) >> (8 * (bb & 3))) & 0xFFu;
              uint32_t sbf = e4m3_pairs_to_bf16x2(sbyte | (sbyte << 16));  // the scale in both halves
              asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(sbf) : "r"(sbf), "r"(0x5F005F00u));  // x 2^63, exact
#pragma unroll
              for (int wi = 0; wi < 2; ++wi)
#pragma unroll
                for (int pi = 0; pi < 4; ++pi)  // k = 16 bb + 8 wi + 2 pi and the next: one column
                  h[(c * 2 + e) * 8 + wi * 4 + pi] = e2m1_pair_to_bf16x2(ws[2 * e + wi] >> (4 * pi), sbf);
            }
          }
          tmem_st32(a_st + static_cast<uint32_t>(q2 * 32), h);
        }
      }
      // x^2 of token `tok` over chunk `sub` of both 64-k atoms of this unit (zero past M and past K)
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const uint4 w = *reinterpret_cast<const uint4*>(sX + s * F::kXStage + half * kD8XStage + a * 2048 +
                                                        (tok >> 3) * 1024 + (tok & 7) * 128 + (sub << 4));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = bf16lo_to_f32(ws[e]), hi = bf16hi_to_f32(ws[e]);
          ss = fmaf(lo, lo, ss);
          ss = fmaf(hi, hi, ss);
        }
      }
      fence_proxy_async_smem();  // the reads above come before the TMA refill this arrival permits
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        // the stage's last unit of this range: its codes are read. A stage of which this range takes one
        // unit of two gets one MMA commit instead of two; one converter warp arrives in its place.
        if (half == F::kUnits - 1 || u == u1 - 1) mbar_arrive(&empty[s]);
        const bool alone = F::kUnits == 2 && ((half == 0 && u == u1 - 1) || (half == 1 && u == u0));
        if (alone && warp == 2) mbar_arrive(&empty[s]);
        mbar_arrive(&afull[b]);
      }
    }
    // A wait that gave up leaves this thread's sum incomplete: it contributes NaN instead, so every output
    // it feeds is NaN (the status word reports the timeout).
    if (!ok) ss = kNaN;
    // the eight threads of a token are eight consecutive lanes
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);

    float v[kD8Tok];
    if (ok) ok = mbar_wait(acc_full, 0, abort_flag);
    if (ok && u1 > u0) {
      tc_fence_after_sync();
      uint32_t r0[16], r1[16], r2[16], r3[16];
      tmem_ld16(tmem_base + lane_base, r0);
      tmem_ld16(tmem_base + lane_base + kD8Tok, r1);
      tmem_ld16(tmem_base + lane_base + 2 * kD8Tok, r2);
      tmem_ld16(tmem_base + lane_base + 3 * kD8Tok, r3);
      tmem_ld_wait();
      reg_fence16(r0);
      reg_fence16(r1);
      reg_fence16(r2);
      reg_fence16(r3);
      // accumulator a belongs to issuer a / kD8AccPer, which wrote it only if this range has a stage for it
      const int nst = u1 - u0;
      const bool w0 = nst > 0 / kD8AccPer, w1 = nst > 1 / kD8AccPer, w2 = nst > 2 / kD8AccPer, w3 = nst > 3 / kD8AccPer;
#pragma unroll
      for (int j = 0; j < kD8Tok; ++j)
        v[j] = ((w0 ? __uint_as_float(r0[j]) : 0.f) + (w1 ? __uint_as_float(r1[j]) : 0.f)) +
               ((w2 ? __uint_as_float(r2[j]) : 0.f) + (w3 ? __uint_as_float(r3[j]) : 0.f));
      if constexpr (FMT == kFmtNvfp4) {
#pragma unroll
        for (int j = 0; j < kD8Tok; ++j) v[j] *= kNvfp4Unscale;  // the A operand held weights x 2^-63: exact
      }
    } else {
      // an empty K range contributes zero; a wait that gave up contributes NaN
#pragma unroll
      for (int j = 0; j < kD8Tok; ++j) v[j] = ok ? 0.f : kNaN;
    }
    if (KSPLIT > 1 && rank != 0) {
      const uint32_t dst = dsmem_addr(part_d + ((rank - 1) * kD8Rows + row) * kD8Tok, 0);
#pragma unroll
      for (int j = 0; j < kD8Tok; j += 4) dsmem_st_v4(dst + j * 4, v[j], v[j + 1], v[j + 2], v[j + 3]);
      if (sub == 0) dsmem_st_f32(dsmem_addr(part_ss + rank * kD8Tok + tok, 0), ss);
    }
    if (KSPLIT > 1) cluster_sync_all();  // the partial sums have reached the leader
    bool writer = rank == 0;  // this CTA writes the slab's output
    if (KSPLIT == 0 && ks > 1) {
      // this range's partials to the workspace, then count the arrival; the last of the slab's ranges
      // to arrive adds them all, range 0 first (the same order whichever range comes last)
      const size_t rec = static_cast<size_t>(slab) * static_cast<size_t>(ks);  // the slab's first record
      float* mine = p.part + ((rec + rank) * kD8Rows + row) * kD8Tok;
      // only the token slots the call has (groups of four below M): the slots past M are never read
#pragma unroll
      for (int j = 0; j < kD8Tok; j += 4)
        if (j < p.M) __stcg(reinterpret_cast<float4*>(mine + j), make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
      if (sub == 0) __stcg(p.part_ss + (rec + rank) * kD8Tok + tok, ss);
      named_bar_sync(1, 128);  // the CTA's partials come before its arrival (barrier, then release)
      if (t == 0) {
        // acquire-release at GPU scope: releases this CTA's partials, and for the last arrival acquires
        // the other ranges' (each released by its own arrival); the barrier below passes that on
        const bool last = atom_add_acq_rel_gpu(p.counters + slab, 1u) == static_cast<unsigned>(ks - 1);
        if (last) st_relaxed_gpu(p.counters + slab, 0u);  // every range has arrived: zero for the next call
        *last_flag = last ? 1 : 0;
      }
      named_bar_sync(1, 128);
      writer = *last_flag != 0;
      if (writer) {
        float tot[kD8Tok];
        float sst = 0.f;
        for (int rr = 0; rr < ks; ++rr) {
          float q[kD8Tok];
          if (rr == static_cast<int>(rank)) {
#pragma unroll
            for (int j = 0; j < kD8Tok; ++j) q[j] = v[j];
          } else {
            const float* src = p.part + ((rec + rr) * kD8Rows + row) * kD8Tok;
#pragma unroll
            for (int j = 0; j < kD8Tok; j += 4) {
              const float4 f = j < p.M ? __ldcg(reinterpret_cast<const float4*>(src + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
              q[j] = f.x, q[j + 1] = f.y, q[j + 2] = f.z, q[j + 3] = f.w;
            }
          }
          const float qs = rr == static_cast<int>(rank) ? ss : (sub == 0 ? __ldcg(p.part_ss + (rec + rr) * kD8Tok + tok) : 0.f);
#pragma unroll
          for (int j = 0; j < kD8Tok; ++j) tot[j] = rr == 0 ? q[j] : tot[j] + q[j];
          sst = rr == 0 ? qs : sst + qs;
        }
#pragma unroll
        for (int j = 0; j < kD8Tok; ++j) v[j] = tot[j];
        ss = sst;
      }
    }
    if (writer) {
      if (KSPLIT > 1) {
        for (int rr = 1; rr < KSPLIT; ++rr) {
#pragma unroll
          for (int j = 0; j < kD8Tok; ++j) v[j] += part_d[((rr - 1) * kD8Rows + row) * kD8Tok + j];
          if (sub == 0) ss += part_ss[rr * kD8Tok + tok];
        }
      }
      if (sub == 0) rs[tok] = 1.0f / sqrtf(ss / static_cast<float>(p.K) + p.eps);
      named_bar_sync(1, 128);
      const int n = n0 + row;
      if (n < p.N) {
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
