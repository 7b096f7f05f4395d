// gemv_kernel.cuh -- decode-shaped I2_S matmul (1 or 2 tokens) on the integer
// ALU, for one or many independent problems in a single persistent launch.
//
// At one or two tokens the ternary contraction ("LLM Quantization
// Paradigms: FP8, AWQ, EXL2 & BitNet b1.58 in 2026", section 5 figure,
// "BitNet b1.58 Ternary Matrix Multiplication") does 4 multiply-adds per
// packed byte per token, far below what the SM's dp4a pipe sustains at HBM
// speed, so it runs as dp4a on registers while the packed weights stream
// through shared memory:
//
//   * Work item = a group of consecutive rows of one problem.  Rows of the
//     I2_S tensor are contiguous, so a group is one contiguous byte range
//     fetched with one 1-D bulk copy into a shared-memory stage.
//   * Each CTA owns one contiguous range of items (items have about the
//     same byte count, so equal ranges balance), so it switches problem only
//     a few times per launch.
//   * Warp 0 (one lane) is the producer: it walks the CTA's items, keeps
//     kStages copies in flight, and when an item starts a new problem it
//     also copies that problem's int8 activations (M x K bytes) into one of
//     two x slots and stages the problem's scales next to them.
//   * Warps 1..12 (1..8 for two tokens) compute, two rows at a time per
//     warp (two independent dependency chains).  Lane l owns packed words l, l+32, ... of every
//     row (so its loads of a row are conflict-free and coalesced) and holds
//     the matching activation words in registers for the whole problem.
//
// Unpack without shifts ("How BitNet's 1-Bit (I2_S) Quantization Works
// Compared to Standard LLM Quantization", Ternary Representation and
// Packing: group g of a byte is bits [7-2g : 6-2g]): word & (3 << (6-2g)) in
// every byte is code_g * 4^(3-g), an unsigned byte in {0, 4^(3-g), 2*4^(3-g)}.
// One dp4a per group and token accumulates sum code*x scaled by 4^(3-g) in
// its own register; at the end of the row the four are rescaled exactly
// (arithmetic shifts of exact multiples), summed, reduced over the warp,
// and sum_k x is subtracted, since w = code - 1.
#pragma once

#include "ptx.cuh"
#include "quant_kernels.cuh"

namespace bitnet {

constexpr int kMaxBatch = 256;

// One independent problem of a batch (all device pointers).
struct BatchProblem {
  const uint8_t* packed;  // I2_S tensor [n, k]
  const float* x;         // fp32 activations [m, k] (read by the batched quantizer)
  int8_t* xq;             // int8 activations [m, k]
  float* xs;              // per-token scales [m]
  float* y;               // [m, n]
  int32_t* acc;           // [m, n] or null
  int32_t n, k;
  int32_t rows_per_item;  // rows of one work item
  int32_t item_start;     // first global work item of this problem
};

template <int CAP>
struct BatchParamsT {
  int32_t count;        // problems
  int32_t m;            // tokens (the same for every problem)
  int32_t total_items;  // work items over all problems
  int32_t pdl;          // 1: activations come from the preceding grid
  BatchProblem p[CAP];
};

struct StageMeta {
  int32_t p, row0, nrows, sw;  // sw: index of the problem switch this item starts, or -1
};

template <int MT, int WPL>
struct GemvCfg {
  static_assert(MT >= 1 && MT <= 2, "tokens");
  static constexpr int kComputeWarps = MT == 1 ? 12 : 8;
  static constexpr int kRowsPerPass = 2;  // rows one warp interleaves
  static constexpr int kThreads = 32 * (kComputeWarps + 1);
  static constexpr int kStageBytes = 32768;
  static constexpr int kStages = 4;
  static constexpr int kMaxK = WPL * 512;  // 32 lanes x WPL words x 16 weights
  static constexpr int kXSlotBytes = MT * kMaxK;
  static constexpr int kBars = 2 * kStages + 4;
  static constexpr size_t kSmemBytes = 128 + static_cast<size_t>(kStages) * kStageBytes +
                                       2 * kXSlotBytes + kBars * 8 + kStages * sizeof(StageMeta) +
                                       2 * 4 * sizeof(float) + 16;
};

__device__ __forceinline__ int dp4a_u8s8(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

template <typename BP>
__device__ __forceinline__ int find_problem(const BP& bp, int item) {
  int lo = 0, hi = bp.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (bp.p[mid].item_start <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

template <int MT, int WPL, int CAP>
__global__ void __launch_bounds__(GemvCfg<MT, WPL>::kThreads, 1)
    i2s_gemv_dp4a_kernel(const __grid_constant__ BatchParamsT<CAP> bp) {
  using C = GemvCfg<MT, WPL>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  uint8_t* stages = smem;
  uint8_t* xslots = smem + S * C::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(xslots + 2 * C::kXSlotBytes);
  StageMeta* meta = reinterpret_cast<StageMeta*>(bars + C::kBars);
  float* xscal = reinterpret_cast<float*>(meta + S);  // per x slot: weight scale, xs[0..MT)
  volatile uint32_t* abort_flag = reinterpret_cast<uint32_t*>(xscal + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto xfull_bar = [&](int j) { return bar0 + 8u * (2 * S + j); };
  auto xempty_bar = [&](int j) { return bar0 + 8u * (2 * S + 2 + j); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), C::kComputeWarps);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(xfull_bar(j), 1);
      mbar_init(xempty_bar(j), C::kComputeWarps);
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();

  const int total = bp.total_items;
  const int m_tokens = bp.m;
  const int item_lo = static_cast<int>(static_cast<int64_t>(total) * blockIdx.x / gridDim.x);
  const int item_hi = static_cast<int>(static_cast<int64_t>(total) * (blockIdx.x + 1) / gridDim.x);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // Weights of the first stages do not depend on the preceding grid:
      // request them before waiting for it.
      // Per stage: the last item whose copy was issued, and whether its
      // phase has received the producer's arrival.
      int issued_item[S];
      bool issued_arrived[S];
#pragma unroll
      for (int s = 0; s < S; ++s) {
        issued_item[s] = -1;
        issued_arrived[s] = false;
      }
      int it = 0;
      for (int item = item_lo; item < item_hi && it < S; ++item, ++it) {
        const int p = find_problem(bp, item);
        const BatchProblem& P = bp.p[p];
        const int row0 = (item - P.item_start) * P.rows_per_item;
        const int nrows = min(P.rows_per_item, P.n - row0);
        const uint32_t bytes = static_cast<uint32_t>(nrows) * static_cast<uint32_t>(P.k >> 2);
        mbar_expect_tx(full_bar(it), bytes);
        bulk_load(smem_u32(stages + it * C::kStageBytes),
                  P.packed + static_cast<size_t>(row0) * (P.k >> 2), bytes, full_bar(it));
        issued_item[it] = it;
      }
      if (bp.pdl) grid_dependency_wait();
      int prev_p = -1, nsw = 0;
      it = 0;
      for (int item = item_lo; item < item_hi; ++item, ++it) {
        const int s = it % S;
        const int p = find_problem(bp, item);
        const BatchProblem& P = bp.p[p];
        const int row0 = (item - P.item_start) * P.rows_per_item;
        const int nrows = min(P.rows_per_item, P.n - row0);
        if (it >= S) {
          if (!mbar_wait(empty_bar(s), ((it / S) - 1) & 1, abort_flag)) break;
          const uint32_t bytes = static_cast<uint32_t>(nrows) * static_cast<uint32_t>(P.k >> 2);
          mbar_expect_tx(full_bar(s), bytes);
          bulk_load(smem_u32(stages + s * C::kStageBytes),
                    P.packed + static_cast<size_t>(row0) * (P.k >> 2), bytes, full_bar(s));
          issued_item[s] = it;
          issued_arrived[s] = false;
        }
        int sw = -1;
        if (p != prev_p) {
          const int slot = nsw & 1;
          if (nsw >= 2 && !mbar_wait(xempty_bar(slot), ((nsw >> 1) - 1) & 1, abort_flag)) break;
          const uint32_t xbytes = static_cast<uint32_t>(m_tokens) * static_cast<uint32_t>(P.k);
          // The scales, ahead of the consumers (published by the arrive below).
          xscal[4 * slot] =
              *reinterpret_cast<const float*>(P.packed + static_cast<size_t>(P.n) * (P.k >> 2));
#pragma unroll
          for (int m = 0; m < MT; ++m) xscal[4 * slot + 1 + m] = (m < m_tokens) ? P.xs[m] : 0.0f;
          mbar_arrive_expect_tx(xfull_bar(slot), xbytes);
          bulk_load(smem_u32(xslots + slot * C::kXSlotBytes), P.xq, xbytes, xfull_bar(slot));
          sw = nsw++;
          prev_p = p;
        }
        StageMeta md;
        md.p = p;
        md.row0 = row0;
        md.nrows = nrows;
        md.sw = sw;
        meta[s] = md;
        mbar_arrive(full_bar(s));  // publishes meta[s]; the phase completes with the bytes
        issued_arrived[s] = true;
      }
      grid_dependents_launch();
      if (*abort_flag) {
        // Let every copy still in flight land before shared memory goes away.
#pragma unroll
        for (int s = 0; s < S; ++s) {
          if (issued_item[s] < 0) continue;
          if (!issued_arrived[s]) mbar_arrive(full_bar(s));
          mbar_wait(full_bar(s), (issued_item[s] / S) & 1, nullptr, kDrainTimeoutNs);
        }
        for (int j = 0; j < 2 && j < nsw; ++j) {
          const int last = nsw - 1 - j;
          mbar_wait(xfull_bar(last & 1), (last >> 1) & 1, nullptr, kDrainTimeoutNs);
        }
      }
    }
    return;
  }

  // ---------------------------------------------------------------- compute
  const int cw = warp - 1;
  if (bp.pdl) grid_dependency_wait();
  uint32_t xr[MT][WPL][4];
  int xsum[MT];
  float xsv[MT];
  float wscale = 0.0f;
  int n = 0, k = 0, wr = 0;
  float* yout = nullptr;
  int32_t* accout = nullptr;
  int it = 0;
  for (int item = item_lo; item < item_hi; ++item, ++it) {
    const int s = it % S;
    if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), (it / S) & 1, abort_flag))) break;
    StageMeta md;
    {
      const volatile int32_t* vm = reinterpret_cast<const volatile int32_t*>(meta + s);
      md.p = vm[0];
      md.row0 = vm[1];
      md.nrows = vm[2];
      md.sw = vm[3];
    }
    if (md.sw >= 0) {
      // A new problem: its activations into registers, then free the slot.
      const int slot = md.sw & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(xfull_bar(slot), (md.sw >> 1) & 1, abort_flag)))
        break;
      const BatchProblem& P = bp.p[md.p];
      n = P.n;
      k = P.k;
      wr = k >> 4;  // packed 32-bit words per row
      yout = P.y;
      accout = P.acc;
      const uint8_t* xsm = xslots + slot * C::kXSlotBytes;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        int sum = 0;
#pragma unroll
        for (int t = 0; t < WPL; ++t) {
          const int j = lane + 32 * t;
          const bool live = (m < m_tokens) && (j < wr);
          // word j of a row covers weights 128*(j/8) + 32*g + 4*(j%8) + {0..3}
          const uint8_t* base = xsm + m * k + (j >> 3) * 128 + (j & 7) * 4;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint32_t v = live ? *reinterpret_cast<const uint32_t*>(base + 32 * g) : 0u;
            xr[m][t][g] = v;
            sum = __dp4a(static_cast<int>(v), 0x01010101, sum);
          }
        }
        xsum[m] = __reduce_add_sync(0xffffffffu, sum);
      }
      wscale = xscal[4 * slot];
#pragma unroll
      for (int m = 0; m < MT; ++m) xsv[m] = xscal[4 * slot + 1 + m];
      __syncwarp();
      if (lane == 0) mbar_arrive(xempty_bar(slot));
    }
    const uint8_t* st = stages + s * C::kStageBytes;
    const int rb = k >> 2;  // bytes per row
    constexpr int R = C::kRowsPerPass;
    for (int r0 = cw * R; r0 < md.nrows; r0 += C::kComputeWarps * R) {
      const uint32_t* row[R];
      bool has[R];
#pragma unroll
      for (int q = 0; q < R; ++q) {
        has[q] = r0 + q < md.nrows;
        row[q] = reinterpret_cast<const uint32_t*>(st + static_cast<size_t>(has[q] ? r0 + q : r0) * rb);
      }
      int a[R][MT][4];
#pragma unroll
      for (int q = 0; q < R; ++q)
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int g = 0; g < 4; ++g) a[q][m][g] = 0;
#pragma unroll
      for (int t = 0; t < WPL; ++t) {
        if (32 * t >= wr) break;  // uniform over the warp
        const int j = lane + 32 * t;
        const bool live = j < wr;
        uint32_t w[R];
#pragma unroll
        for (int q = 0; q < R; ++q) w[q] = (live && has[q]) ? row[q][j] : 0u;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint32_t mask = 0x03030303u << (6 - 2 * g);
#pragma unroll
          for (int q = 0; q < R; ++q) {
            const uint32_t v = w[q] & mask;
#pragma unroll
            for (int m = 0; m < MT; ++m) a[q][m][g] = dp4a_u8s8(v, xr[m][t][g], a[q][m][g]);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < R; ++q) {
        const int64_t nn = static_cast<int64_t>(md.row0) + r0 + q;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int part = (a[q][m][0] >> 6) + (a[q][m][1] >> 4) + (a[q][m][2] >> 2) + a[q][m][3];
          const int dot = __reduce_add_sync(0xffffffffu, part) - xsum[m];
          if (has[q] && lane == m && m < m_tokens) {
            yout[m * static_cast<int64_t>(n) + nn] =
                __fmul_rn(__fmul_rn(__int2float_rn(dot), xsv[m]), wscale);
            if (accout != nullptr) accout[m * static_cast<int64_t>(n) + nn] = dot;
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
  }
}

// Per-token absmax quantization of every problem's activations: one CTA per
// (problem, token) row, the same arithmetic as act_quant_kernel.
template <int CAP>
__global__ void __launch_bounds__(256) act_quant_batched_kernel(
    const __grid_constant__ BatchParamsT<CAP> bp) {
  grid_dependency_wait();
  grid_dependents_launch();
  __shared__ float red[32];
  const int p = blockIdx.x / bp.m;
  const int m = blockIdx.x % bp.m;
  const BatchProblem& P = bp.p[p];
  quantize_row(P.x + static_cast<int64_t>(m) * P.k, P.k, P.xq + static_cast<int64_t>(m) * P.k,
               P.xs + m, red);
}

}  // namespace bitnet
