// mma_kernel.cuh -- the I2_S ternary x int8 matmul on the sm_100a tensor
// cores (tcgen05.mma kind::i8, int32 accumulators in tensor memory).
//
// The contraction acc[m,n] = sum_k w[n,k]*xq[m,k] of "LLM Quantization
// Paradigms: FP8, AWQ, EXL2 & BitNet b1.58 in 2026" (section 5 figure,
// "BitNet b1.58 Ternary Matrix Multiplication") is exact in integers, so it
// runs as a dense int8 MMA: the packed 2-bit weights are expanded once per
// tile to int8 (the unpack of "How BitNet's 1-Bit (I2_S) Quantization Works
// Compared to Standard LLM Quantization", How I2_S Kernels Process the
// Format) and contracted with the int8 activations.
//
// Tile ("swap-AB"): MMA M = 128 weight rows (operand A, held in TMEM), MMA
// N = T tokens (operand B, Xq rows, K-major in shared memory), so a decode
// batch of 1..64 tokens still fills the 128-row MMA.  One CTA computes one
// 128 x T output tile over the whole K.
//
// Roles (192 threads):
//   warp 0     TMA producer: per stage, one 128-row x 128-byte box of packed
//              weights (512 k, four I2_S blocks) with the 128-byte swizzle,
//              and one T x 128-byte box of Xq per I2_S block.
//   warp 1     TMEM allocator and MMA issuer (one thread).
//   warps 2-5  unpackers, then the epilogue.  Thread r (= TMEM lane r) owns
//              weight row r of the tile: it reads its row's 32 bytes of one
//              block from shared memory, expands them into 4 groups x 32
//              int8 values and stores them as 32 TMEM columns (one A slot).
//
// Unpack: the 32-bit word made of bytes 4i..4i+3 of a block, shifted right
// by 6-2g and masked with 0x03030303, is the four codes of weights
// 32g+4i .. 32g+4i+3 in byte order, i.e. exactly one TMEM column of the A
// operand for the MMA over k = 32g .. 32g+31.  Two variants:
//   kCodes = true:  A holds the unsigned codes c = w+1 (two ALU ops per four
//     weights) and every MMA is followed by one MMA with a constant A of -1,
//     so D = sum (w+1) x - sum x = sum w x.  Used for decode, where the
//     tensor pipe is idle and ALU issue is the scarce resource.
//   kCodes = false: A holds w itself (three more ALU ops per four weights)
//     and no correction MMA is needed.  Used for prefill, where the tensor
//     pipe is the bound and the unpack is amortised over T tokens.
//
// Pipelines: `full/empty` over the shared-memory stages (TMA -> unpack + MMA),
// `afull/aempty` over four TMEM A slots (unpack -> MMA), `dfull` for the
// accumulator (MMA -> epilogue).  Every wait is bounded (ptx.cuh).
#pragma once

#include "ptx.cuh"

namespace bitnet {

struct MmaParams {
  const uint8_t* packed;  // I2_S tensor; the fp32 scale sits at packed + n*k/4
  const float* xs;        // per-token activation scales [m]
  float* y;               // [m, n] fp32
  int32_t* acc;           // [m, n] int32 or null
  int64_t n, k, m;
  int pdl;  // 1: activations are written by the preceding grid (wait for it)
};

constexpr uint32_t round32(uint32_t v) { return (v + 31u) & ~31u; }
constexpr uint32_t pow2_at_least(uint32_t v) {
  uint32_t p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <int T, bool kCodes>
struct MmaCfg {
  static_assert(T % 16 == 0 && T >= 16 && T <= 128, "token tile");
  static constexpr int kRows = 128;                     // MMA M
  static constexpr int kWTileBytes = kRows * 128;       // packed box: 128 rows x 128 B
  static constexpr int kXBoxBytes = T * 128;            // Xq box: T rows x 128 B
  static constexpr int kStageBytes = kWTileBytes + 4 * kXBoxBytes;
  static constexpr int kStages = (T <= 16) ? 4 : (T <= 32 ? 3 : 2);
  static constexpr int kASlots = 4;
  static constexpr uint32_t kDCol = 0;
  static constexpr uint32_t kNegCol = round32(T);
  static constexpr uint32_t kACol = kCodes ? kNegCol + 32u : round32(T);
  static constexpr uint32_t kTmemCols = pow2_at_least(kACol + 32u * kASlots);
  static constexpr int kNumBars = 2 * kStages + 2 * kASlots + 1;
  static constexpr size_t kSmemBytes =
      1024 /*alignment slack*/ + static_cast<size_t>(kStages) * kStageBytes + kNumBars * 8 + 16;
  static constexpr uint32_t kIdescA = idesc_i8(128, T, !kCodes, true);
  static constexpr uint32_t kIdescNeg = idesc_i8(128, T, true, true);
};

template <bool kCodes>
__device__ __forceinline__ uint32_t unpack_word(uint32_t w, int g) {
  const uint32_t c = (w >> (6 - 2 * g)) & 0x03030303u;
  if (kCodes) return c;
  // c in {0,1,2} per byte -> c - 1 per byte; the 0x80 bias keeps every byte
  // from borrowing out of its neighbour.
  return ((c | 0x80808080u) - 0x01010101u) ^ 0x80808080u;
}

template <int T, bool kCodes>
__global__ void __launch_bounds__(192) i2s_mma_kernel(const __grid_constant__ CUtensorMap tm_w,
                                                      const __grid_constant__ CUtensorMap tm_x,
                                                      const MmaParams p) {
  using C = MmaCfg<T, kCodes>;
  constexpr int S = C::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint32_t* misc = reinterpret_cast<uint32_t*>(bars + C::kNumBars);  // [0] tmem, [1] abort
  volatile uint32_t* abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * C::kRows;
  const int64_t tok0 = static_cast<int64_t>(blockIdx.y) * T;
  const int n_blocks = static_cast<int>(p.k / 128);
  const int n_chunks = (n_blocks + 3) / 4;

  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto afull_bar = [&](int t) { return bar0 + 8u * (2 * S + t); };
  auto aempty_bar = [&](int t) { return bar0 + 8u * (2 * S + C::kASlots + t); };
  const uint32_t dfull_bar = bar0 + 8u * (2 * S + 2 * C::kASlots);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 4 + 1);  // four unpack warps + one MMA commit
    }
    for (int t = 0; t < C::kASlots; ++t) {
      mbar_init(afull_bar(t), 4);
      mbar_init(aempty_bar(t), 1);
    }
    mbar_init(dfull_bar, 1);
    misc[1] = 0u;
    fence_mbar_init();
    prefetch_tensormap(&tm_w);
    prefetch_tensormap(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int pre = n_chunks < S ? n_chunks : S;
      // Weights first: they do not depend on the preceding grid, so their
      // loads overlap its tail when launched as a dependent grid.
      for (int kc = 0; kc < pre; ++kc) {
        const int nb = min(4, n_blocks - 4 * kc);
        mbar_arrive_expect_tx(full_bar(kc), C::kWTileBytes + nb * C::kXBoxBytes);
        tma_load_2d(smem_u32(smem + kc * C::kStageBytes), &tm_w, kc * 128,
                    static_cast<int32_t>(row0), full_bar(kc));
      }
      if (p.pdl) grid_dependency_wait();
      int issued = 0;
      for (int kc = 0; kc < n_chunks; ++kc) {
        const int s = kc % S;
        const int nb = min(4, n_blocks - 4 * kc);
        uint8_t* st = smem + s * C::kStageBytes;
        if (kc >= pre) {
          if (!mbar_wait(empty_bar(s), ((kc / S) - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(full_bar(s), C::kWTileBytes + nb * C::kXBoxBytes);
          tma_load_2d(smem_u32(st), &tm_w, kc * 128, static_cast<int32_t>(row0), full_bar(s));
        }
        for (int q = 0; q < nb; ++q)
          tma_load_2d(smem_u32(st + C::kWTileBytes + q * C::kXBoxBytes), &tm_x,
                      kc * 512 + q * 128, static_cast<int32_t>(tok0), full_bar(s));
        issued = kc + 1;
      }
      grid_dependents_launch();
      if (*abort_flag) {
        // A break can only happen at kc >= pre, so chunks [0, issued) have all
        // their loads in flight.  Let the last one of each stage land before
        // the CTA's shared memory goes away.
        const int first = issued > S ? issued - S : 0;
        for (int kc = first; kc < issued; ++kc)
          mbar_wait(full_bar(kc % S), (kc / S) & 1, nullptr, kDrainTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int blk = 0;
      bool ok = true;
      for (int kc = 0; kc < n_chunks && ok; ++kc) {
        const int s = kc % S;
        ok = mbar_wait(full_bar(s), (kc / S) & 1, abort_flag);
        if (!ok) break;
        const int nb = min(4, n_blocks - 4 * kc);
        const uint32_t xbase = smem_u32(smem + s * C::kStageBytes + C::kWTileBytes);
        for (int bi = 0; bi < nb; ++bi, ++blk) {
          const int t = blk & 3;
          ok = mbar_wait(afull_bar(t), (blk >> 2) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t xb = xbase + bi * C::kXBoxBytes;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            // K step g of this block: bytes 32g..32g+31 of each 128-byte Xq row.
            const uint64_t bdesc = smem_desc_sw128(xb + 32u * g);
            mma_i8_tmem_a(tmem + C::kDCol, tmem + C::kACol + 32u * t + 8u * g, bdesc, C::kIdescA,
                          (blk | g) != 0 ? 1u : 0u);
            if (kCodes) mma_i8_tmem_a(tmem + C::kDCol, tmem + C::kNegCol, bdesc, C::kIdescNeg, 1u);
          }
          tc_commit(aempty_bar(t));
        }
        if (ok) tc_commit(empty_bar(s));
      }
      tc_commit(dfull_bar);
      // Our MMAs must be finished before TMEM is released.
      mbar_wait(dfull_bar, 0, nullptr, ok ? kWaitTimeoutNs : kDrainTimeoutNs);
    }
  } else {
    // ------------------------------------------------ unpack, then epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = true;
    if (kCodes) {
      uint32_t neg[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) neg[i] = 0xFFFFFFFFu;  // int8 -1 x 4
      tmem_st_32x32b_x8(tmem + lane_base + C::kNegCol, neg);
    }
    int blk = 0;
    for (int kc = 0; kc < n_chunks && ok; ++kc) {
      const int s = kc % S;
      ok = __all_sync(0xffffffffu, mbar_wait(full_bar(s), (kc / S) & 1, abort_flag));
      if (!ok) break;
      const int nb = min(4, n_blocks - 4 * kc);
      const uint8_t* wrow = smem + s * C::kStageBytes + r * 128;
      for (int bi = 0; bi < nb; ++bi, ++blk) {
        const int t = blk & 3;
        // The box was written with the 128-byte swizzle: 16-byte chunk c of
        // row r sits at chunk c ^ (r % 8).
        const uint4 c0 = *reinterpret_cast<const uint4*>(wrow + (((2 * bi) ^ (r & 7)) << 4));
        const uint4 c1 = *reinterpret_cast<const uint4*>(wrow + (((2 * bi + 1) ^ (r & 7)) << 4));
        const uint32_t wv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        uint32_t a[32];
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
          for (int i = 0; i < 8; ++i) a[8 * g + i] = unpack_word<kCodes>(wv[i], g);
        if (blk >= C::kASlots) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(aempty_bar(t), ((blk >> 2) - 1) & 1, abort_flag));
          if (!ok) break;
        }
        tc_fence_after();
        tmem_st_32x32b_x32(tmem + lane_base + C::kACol + 32u * t, a);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(afull_bar(t));
      }
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(empty_bar(s));
    }
    // Epilogue: y = ((float)acc * xs[m]) * s, token-major rows.
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dfull_bar, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      if (p.pdl) grid_dependency_wait();
      const float s = *reinterpret_cast<const float*>(p.packed + p.n * p.k / 4);
      const int64_t n = row0 + r;
#pragma unroll 1
      for (int c0 = 0; c0 < T; c0 += 16) {
        if (tok0 + c0 >= p.m) break;  // warp-uniform
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lane_base + C::kDCol + c0, v);
        tmem_ld_wait();
        if (n < p.n) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int64_t tok = tok0 + c0 + j;
            if (tok < p.m) {
              const int32_t a = static_cast<int32_t>(v[j]);
              p.y[tok * p.n + n] = __fmul_rn(__fmul_rn(__int2float_rn(a), __ldg(p.xs + tok)), s);
              if (p.acc != nullptr) p.acc[tok * p.n + n] = a;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace bitnet
