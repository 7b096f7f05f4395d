// mma_kernel.cuh -- the I2_S ternary x int8 matmul on the sm_100a tensor
// cores (tcgen05.mma kind::i8, int32 accumulators in tensor memory), one
// persistent launch over one or many independent problems.
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
// batch of 3..64 tokens still fills the 128-row MMA.  A work item is one
// 128 x T output tile over the whole K.  Items are numbered problem by
// problem, token tile by token tile, row tile by row tile; each CTA owns one
// contiguous range of items balanced by their 512-wide K chunks, and streams
// through it without stopping between items.
//
// Roles (320 threads):
//   warp 0     TMA producer: per chunk one 128-row x 128-byte box of packed
//              weights (512 k, four I2_S blocks) with the 128-byte swizzle,
//              and one T x 128-byte box of Xq per I2_S block.
//   warp 1     TMEM allocator and MMA issuer (one thread).
//   warps 2-5  unpackers: thread r (= TMEM lane r) owns weight row r of the
//              tile; per block it expands its row's 32 bytes into 4 groups x
//              32 int8 values and stores them as 32 TMEM columns (one A
//              slot).  In code mode they also add up each token's int8
//              activations from the staged Xq boxes.
//   warps 6-9  epilogue: y = ((float)acc * xs[m]) * s from the accumulator,
//              token-major, while the next tile's MMAs run into the other
//              accumulator buffer.
//
// Unpack: the 32-bit word made of bytes 4i..4i+3 of a block, shifted right
// by 6-2g and masked with 0x03030303, is the four codes of weights
// 32g+4i .. 32g+4i+3 in byte order, i.e. one TMEM column of the A operand
// for the MMA over k = 32g .. 32g+31.  Two variants:
//   kCodes = true:  A holds the unsigned codes c = w+1 (two ALU ops per four
//     weights); the epilogue subtracts sum_k x, which the unpackers add up
//     from the Xq boxes on their way through shared memory.  For decode,
//     where ALU issue is scarce and the MMAs are small.
//   kCodes = false: A holds w itself (three more ALU ops per four weights).
//     For prefill, where the unpack is amortised over 128 tokens.
//
// Pipelines: full/empty over the shared-memory stages (TMA -> unpack + MMA),
// afull/aempty over four TMEM A slots handed over in pairs (unpack -> MMA),
// dfull/dempty over two
// accumulator buffers (MMA + unpackers -> epilogue -> MMA).  Every wait is
// bounded (ptx.cuh); there are no named barriers, so a timed-out wait can
// never leave another warp stuck.
#pragma once

#include "ptx.cuh"

namespace bitnet {

constexpr uint32_t round32(uint32_t v) { return (v + 31u) & ~31u; }
constexpr uint32_t pow2_at_least(uint32_t v) {
  uint32_t p = 32;
  while (p < v) p <<= 1;
  return p;
}

struct MmaProblem {
  const uint8_t* packed;  // I2_S tensor; the fp32 scale sits at packed + n*k/4
  const float* xs;        // per-token activation scales [m]
  float* y;               // [m, n] fp32
  int32_t* acc;           // [m, n] int32 or null
  int32_t n, k;
  int32_t item_start;     // first global item of this problem
  int32_t chunk_start;    // first global 512-wide K chunk of this problem
};

template <int CAP>
struct MmaParamsT {
  int32_t count;         // problems
  int32_t m;             // tokens (the same for every problem)
  int32_t total_items;   // output tiles over all problems
  int32_t total_chunks;  // K chunks over all items
  int32_t pdl;           // 1: activations come from the preceding grid
  int32_t pad[11];
  CUtensorMap tw[CAP];   // packed bytes as [n rows, k/4 bytes], box 128 x 128
  CUtensorMap tx[CAP];   // Xq as [m rows, k bytes], box 128 x T
  MmaProblem p[CAP];
};

template <int T, bool kCodes>
struct MmaCfg {
  static_assert(T % 16 == 0 && T >= 16 && T <= 128, "token tile");
  static constexpr int kRows = 128;                     // MMA M
  static constexpr int kThreads = 320;
  static constexpr int kWTileBytes = kRows * 128;       // packed box: 128 rows x 128 B
  static constexpr int kXBoxBytes = T * 128;            // Xq box: T rows x 128 B
  static constexpr int kStageBytes = kWTileBytes + 4 * kXBoxBytes;
  static constexpr int kStages = (T <= 16) ? 4 : (T <= 32 ? 3 : 2);
  static constexpr int kCtasPerSm = (T <= 64) ? 2 : 1;
  static constexpr int kASlots = 4;
  static constexpr int kAGroup = 2;  // A slots handed over per handshake (two groups in flight)
  static constexpr uint32_t kDCols = round32(T);        // one accumulator buffer
  static constexpr uint32_t kACol = 2 * kDCols;         // A slots after both buffers
  static constexpr uint32_t kTmemCols = pow2_at_least(kACol + 32u * kASlots);
  static constexpr int kNumBars = 2 * kStages + 2 * kASlots + 4;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes +
                                       kNumBars * 8 + 2 * T * 4 + 16;
  static constexpr uint32_t kIdesc = idesc_i8(128, T, !kCodes, true);
};

template <bool kCodes>
__device__ __forceinline__ uint32_t unpack_word(uint32_t w, int g) {
  const uint32_t c = (w >> (6 - 2 * g)) & 0x03030303u;
  if (kCodes) return c;
  // c in {0,1,2} per byte -> c - 1 per byte; the 0x80 bias keeps every byte
  // from borrowing out of its neighbour.
  return ((c | 0x80808080u) - 0x01010101u) ^ 0x80808080u;
}

template <typename BP>
__device__ __forceinline__ int mma_find_problem(const BP& bp, int item) {
  int lo = 0, hi = bp.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (bp.p[mid].item_start <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// First item whose first chunk is at or after global chunk `target`.
template <typename BP>
__device__ __forceinline__ int mma_first_item_at(const BP& bp, int target) {
  if (target >= bp.total_chunks) return bp.total_items;
  int lo = 0, hi = bp.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (bp.p[mid].chunk_start <= target) lo = mid;
    else hi = mid - 1;
  }
  const MmaProblem& P = bp.p[lo];
  const int nk = (P.k + 511) >> 9;
  const int next = (lo + 1 < bp.count) ? bp.p[lo + 1].item_start : bp.total_items;
  const int items = next - P.item_start;
  const int off = (target - P.chunk_start + nk - 1) / nk;
  return off >= items ? next : P.item_start + off;
}

// Problem, row tile and token tile of an item.
template <typename BP>
__device__ __forceinline__ void mma_item(const BP& bp, int item, int T, int* p, int* rt, int* tt) {
  *p = mma_find_problem(bp, item);
  const MmaProblem& P = bp.p[*p];
  const int row_tiles = (P.n + 127) >> 7;
  const int local = item - P.item_start;
  *tt = local / row_tiles;
  *rt = local - *tt * row_tiles;
  (void)T;
}

template <int T, bool kCodes, int CAP>
__global__ void __launch_bounds__(320, MmaCfg<T, kCodes>::kCtasPerSm)
    i2s_mma_kernel(const __grid_constant__ MmaParamsT<CAP> bp) {
  using C = MmaCfg<T, kCodes>;
  constexpr int S = C::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  int32_t* xsum_smem = reinterpret_cast<int32_t*>(bars + C::kNumBars);  // [2][T]
  uint32_t* misc = reinterpret_cast<uint32_t*>(xsum_smem + 2 * T);     // [0] tmem, [1] abort
  volatile uint32_t* abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tokens = bp.m;

  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto afull_bar = [&](int t) { return bar0 + 8u * (2 * S + t); };
  auto aempty_bar = [&](int t) { return bar0 + 8u * (2 * S + C::kASlots + t); };
  auto dfull_bar = [&](int b) { return bar0 + 8u * (2 * S + 2 * C::kASlots + b); };
  auto dempty_bar = [&](int b) { return bar0 + 8u * (2 * S + 2 * C::kASlots + 2 + b); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 4 + 1);  // four unpack warps + one MMA commit
    }
    for (int t = 0; t < C::kASlots; ++t) {
      mbar_init(afull_bar(t), 4);
      mbar_init(aempty_bar(t), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(dfull_bar(b), kCodes ? 1 + 4 : 1);  // MMA commit (+ the unpackers' sums)
      mbar_init(dempty_bar(b), 4);                  // four epilogue warps
    }
    misc[1] = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  const int64_t tc = bp.total_chunks;
  const int item_lo = mma_first_item_at(bp, static_cast<int>(tc * blockIdx.x / gridDim.x));
  const int item_hi = mma_first_item_at(bp, static_cast<int>(tc * (blockIdx.x + 1) / gridDim.x));

  // Launch chaining: every thread but the producer signals the next grid
  // once it has waited for this grid's inputs (at once when the launch reads
  // nothing the preceding grid writes); the producer does so after its own
  // lazy wait, and waits once more for the preceding grid before it exits.
  // The stages every role consumes carry activations, which the producer
  // requests only after its wait, so the other roles lose nothing by waiting.
  if (warp != 0 || lane != 0) {
    if (bp.pdl) grid_dependency_wait();
    grid_dependents_launch();
  }

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      // The weights of the first stages do not depend on the preceding grid:
      // request them before waiting for it.  Each stage's barrier expects
      // the weight and activation bytes together.
      int issued = 0;
      bool waited = (bp.pdl == 0);
      if (waited) grid_dependents_launch();
      bool ok = true;
      int pre_item = item_lo, pre_kc = 0;  // chunk cursor of the activation loads
      auto chunk_blocks = [&](const MmaProblem& P, int kc) { return min(4, (P.k >> 7) - 4 * kc); };
      auto issue_x = [&](int s, int item, int kc) {
        int p, rt, tt;
        mma_item(bp, item, T, &p, &rt, &tt);
        const MmaProblem& P = bp.p[p];
        const int nb = chunk_blocks(P, kc);
        uint8_t* st = smem + s * C::kStageBytes;
        for (int q = 0; q < nb; ++q)
          tma_load_2d(smem_u32(st + C::kWTileBytes + q * C::kXBoxBytes), &bp.tx[p],
                      kc * 512 + q * 128, tt * T, full_bar(s));
      };
      for (int item = item_lo; item < item_hi && ok; ++item) {
        int p, rt, tt;
        mma_item(bp, item, T, &p, &rt, &tt);
        const MmaProblem& P = bp.p[p];
        prefetch_tensormap(&bp.tw[p]);
        prefetch_tensormap(&bp.tx[p]);
        const int nk = (P.k + 511) >> 9;
        for (int kc = 0; kc < nk; ++kc) {
          const int s = issued % S;
          if (issued >= S) {
            if (!waited) {
              grid_dependency_wait();
              grid_dependents_launch();
              waited = true;
              for (int i = 0; i < S; ++i) {  // activations of the stages issued so far
                issue_x(i, pre_item, pre_kc);
                int pp, r2, t2;
                mma_item(bp, pre_item, T, &pp, &r2, &t2);
                if (++pre_kc == ((bp.p[pp].k + 511) >> 9)) {
                  pre_kc = 0;
                  ++pre_item;
                }
              }
            }
            if (!mbar_wait(empty_bar(s), ((issued / S) - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
          }
          const int nb = chunk_blocks(P, kc);
          mbar_arrive_expect_tx(full_bar(s), C::kWTileBytes + nb * C::kXBoxBytes);
          tma_load_2d(smem_u32(smem + s * C::kStageBytes), &bp.tw[p], kc * 128, rt * 128,
                      full_bar(s));
          if (waited) issue_x(s, item, kc);
          ++issued;
        }
      }
      if (!waited && ok) {
        grid_dependency_wait();
        grid_dependents_launch();
        waited = true;
        for (int i = 0; i < issued; ++i) {
          issue_x(i, pre_item, pre_kc);
          int pp, r2, t2;
          mma_item(bp, pre_item, T, &pp, &r2, &t2);
          if (++pre_kc == ((bp.p[pp].k + 511) >> 9)) {
            pre_kc = 0;
            ++pre_item;
          }
        }
      }
      // This CTA does not finish before the preceding grid has, so that the
      // completion of any grid in a chain implies that of all before it.
      grid_dependency_wait();
      if (*abort_flag) {
        // Let the copies already issued land before shared memory goes away
        // (a stage whose activations were never requested cannot complete;
        // its weight copy has landed by the end of this bounded wait).
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait(full_bar(i % S), (i / S) & 1, nullptr, kDrainTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      int chunk = 0, blk = 0, ii = 0;
      for (int item = item_lo; item < item_hi && ok; ++item, ++ii) {
        int p, rt, tt;
        mma_item(bp, item, T, &p, &rt, &tt);
        const MmaProblem& P = bp.p[p];
        const int b = ii & 1;
        if (ii >= 2 && !mbar_wait(dempty_bar(b), ((ii >> 1) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + b * C::kDCols;
        const int nk = (P.k + 511) >> 9;
        bool first = true;
        for (int kc = 0; kc < nk && ok; ++kc, ++chunk) {
          const int s = chunk % S;
          if (!mbar_wait(full_bar(s), (chunk / S) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int nb = min(4, (P.k >> 7) - 4 * kc);
          const uint32_t xbase = smem_u32(smem + s * C::kStageBytes + C::kWTileBytes);
          for (int bi = 0; bi < nb; ++bi, ++blk) {
            const int t = blk & 3;
            const int group = blk / C::kAGroup;
            if (blk % C::kAGroup == 0) {
              if (!mbar_wait(afull_bar(group & 1), (group >> 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            const uint32_t xb = xbase + bi * C::kXBoxBytes;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              // K step g of this block: bytes 32g..32g+31 of each 128-byte Xq row.
              mma_i8_tmem_a(dcol, tmem + C::kACol + 32u * t + 8u * g,
                            smem_desc_sw128(xb + 32u * g), C::kIdesc, first ? 0u : 1u);
              first = false;
            }
            if (blk % C::kAGroup == C::kAGroup - 1) tc_commit(aempty_bar(group & 1));
          }
          if (ok) tc_commit(empty_bar(s));
        }
        if (ok) tc_commit(dfull_bar(b));
      }
      // Our MMAs must be finished before TMEM is released.
      const int last = ii - 1;
      if (last >= 0)
        mbar_wait(dfull_bar(last & 1), (last >> 1) & 1, nullptr,
                  ok ? kWaitTimeoutNs : kDrainTimeoutNs);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ unpack
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int ut = (warp - 2) * 32 + lane;  // 0..127 among the unpackers
    bool ok = true;
    int chunk = 0, blk = 0, ii = 0;
    // A slots are handed over in pairs (C::kAGroup blocks): one store wait
    // and one arrival per pair, and one commit per pair on the MMA side.
    auto hand_over = [&](int group) {
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(afull_bar(group & 1));
    };
    for (int item = item_lo; item < item_hi && ok; ++item, ++ii) {
      int p, rt, tt;
      mma_item(bp, item, T, &p, &rt, &tt);
      const MmaProblem& P = bp.p[p];
      const int nk = (P.k + 511) >> 9;
      int xacc[T / 16];  // code mode: token sums of this thread's Xq chunks
#pragma unroll
      for (int i = 0; i < T / 16; ++i) xacc[i] = 0;
      for (int kc = 0; kc < nk && ok; ++kc, ++chunk) {
        const int s = chunk % S;
        ok = __all_sync(0xffffffffu, mbar_wait(full_bar(s), (chunk / S) & 1, abort_flag));
        if (!ok) break;
        const int nb = min(4, (P.k >> 7) - 4 * kc);
        const uint8_t* stage = smem + s * C::kStageBytes;
        const uint8_t* wrow = stage + r * 128;
        for (int bi = 0; bi < nb; ++bi, ++blk) {
          const int t = blk & 3;
          if (kCodes) {
            // Token sums: the box holds T rows x 8 chunks of 16 bytes; this
            // thread adds chunk (ut % 8) of rows ut / 8 + 16 i.  The swizzle
            // only permutes chunks inside a row, so any chunk order will do.
            const uint8_t* xb = stage + C::kWTileBytes + bi * C::kXBoxBytes;
#pragma unroll
            for (int i = 0; i < T / 16; ++i) {
              const uint4 v =
                  *reinterpret_cast<const uint4*>(xb + (ut / 8 + 16 * i) * 128 + (ut % 8) * 16);
              int a = xacc[i];
              a = __dp4a(static_cast<int>(v.x), 0x01010101, a);
              a = __dp4a(static_cast<int>(v.y), 0x01010101, a);
              a = __dp4a(static_cast<int>(v.z), 0x01010101, a);
              a = __dp4a(static_cast<int>(v.w), 0x01010101, a);
              xacc[i] = a;
            }
          }
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
          const int group = blk / C::kAGroup;
          if (blk % C::kAGroup == 0 && group >= 2) {
            // The pair of slots this group reuses has been read by its MMAs.
            ok = __all_sync(0xffffffffu,
                            mbar_wait(aempty_bar(group & 1), ((group >> 1) - 1) & 1, abort_flag));
            if (!ok) break;
          }
          tc_fence_after();
          tmem_st_32x32b_x32(tmem + lane_base + C::kACol + 32u * t, a);
          if (blk % C::kAGroup == C::kAGroup - 1) hand_over(group);
        }
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(empty_bar(s));
      }
      if (kCodes && ok) {
        // Sum the 8 chunk threads of each row, publish with the dfull arrival.
        const int b = ii & 1;
        if (ii >= 2)
          ok = __all_sync(0xffffffffu, mbar_wait(dempty_bar(b), ((ii >> 1) - 1) & 1, abort_flag));
        if (!ok) break;
#pragma unroll
        for (int i = 0; i < T / 16; ++i) {
          int v = xacc[i];
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          if ((ut & 7) == 0) xsum_smem[b * T + ut / 8 + 16 * i] = v;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(dfull_bar(b));
      }
    }
    if (ok && blk % C::kAGroup != 0) hand_over(blk / C::kAGroup);  // a last, partial pair
    tmem_st_wait();  // no store of this thread outlives it
  } else {
    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int ii = 0;
    for (int item = item_lo; item < item_hi; ++item, ++ii) {
      int p, rt, tt;
      mma_item(bp, item, T, &p, &rt, &tt);
      const MmaProblem& P = bp.p[p];
      const int b = ii & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(dfull_bar(b), (ii >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const float s = *reinterpret_cast<const float*>(P.packed + static_cast<int64_t>(P.n) * (P.k >> 2));
      const int64_t n = static_cast<int64_t>(rt) * 128 + r;
      const int64_t tok0 = static_cast<int64_t>(tt) * T;
#pragma unroll 1
      for (int c0 = 0; c0 < T; c0 += 16) {
        if (tok0 + c0 >= m_tokens) break;  // warp-uniform
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lane_base + b * C::kDCols + c0, v);
        tmem_ld_wait();
        if (n < P.n) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int64_t tok = tok0 + c0 + j;
            if (tok < m_tokens) {
              int32_t a = static_cast<int32_t>(v[j]);
              if (kCodes) a -= xsum_smem[b * T + c0 + j];
              P.y[tok * P.n + n] = __fmul_rn(__fmul_rn(__int2float_rn(a), __ldg(P.xs + tok)), s);
              if (P.acc != nullptr) P.acc[tok * P.n + n] = a;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dempty_bar(b));
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
