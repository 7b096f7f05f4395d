// gemv_kernel.cuh -- decode-shaped I2_S matmul (1 or 2 tokens) on the integer
// ALU, for one or many independent problems in a single persistent launch.
// Two activation-slot sizes: K <= 8192 (one or two tokens, 3 or 2 CTAs per
// SM) and, for one token, K <= 30720 (2 CTAs per SM).
//
// At one or two tokens the ternary contraction ("LLM Quantization
// Paradigms: FP8, AWQ, EXL2 & BitNet b1.58 in 2026", section 5 figure,
// "BitNet b1.58 Ternary Matrix Multiplication") does 4 multiply-adds per
// packed byte per token, well within what dp4a sustains at HBM speed, so it
// runs on the ALU while the packed weights stream through shared memory:
//
//   * Work item = a tile of 128 rows of one problem over the whole K.
//     The tile streams in stages of one TMA box of 128 rows x 128 bytes
//     (512 weights of each row) written with the 128-byte swizzle.
//   * Each CTA owns one contiguous range of items, balanced by stages, so it
//     changes problem only a few times per launch.  With a work counter
//     (batched calls with a workspace) the ranges cover the first part of
//     the launch's stages and the remaining items are handed out one at a
//     time as CTAs become free, which evens out when the CTAs finish.
//     Warp 0 (one lane) is the producer; on a change of problem it also
//     copies the problem's int8 activations (M x K bytes) into one of two x
//     slots and stages the two scales next to them.  Weights are streamed
//     with an evict-first L2 policy, so the activations stay in L2.
//   * Warps 1..4 compute; warp w owns rows 32w..32w+31 of the tile.  Within
//     a box, lane (rs, cp) = (lane / 4, lane % 4) owns I2_S block cp (32
//     bytes, 128 weights) of the 4 rows 32w + rs + 8i, i = 0..3.  It loads
//     the 128 activation bytes of its block into registers once per box and
//     reuses them for its 4 rows, so shared-memory traffic is one read of
//     each weight byte plus a quarter of an activation byte per weight byte
//     (a broadcast read costs as many wavefronts as a plain one).  The
//     128-byte swizzle makes the 8 lanes of each quarter-warp hit 8
//     different bank groups for the weights; for the activations, lane cp
//     visits the four groups starting at group cp, so the four blocks' reads
//     of one instruction fall in four different 32-byte bank groups.  At the
//     end of a tile the 4 lanes of a row add their partial sums with two
//     shuffles.
//
// Launch chaining (programmatic dependent launch): every thread signals the
// next grid in the stream as soon as it has waited for its own inputs (at
// once when the launch reads nothing the preceding grid writes), so the next
// launch's CTAs take over SMs as soon as this launch's CTAs leave, and one
// thread per CTA waits for the preceding grid before the CTA exits, so that
// a grid never completes before the one it follows.
//
// Unpack without shifts ("How BitNet's 1-Bit (I2_S) Quantization Works
// Compared to Standard LLM Quantization", Ternary Representation and
// Packing: group g of a byte is bits [7-2g : 6-2g]): word & (3 << (6-2g)) in
// every byte is code_g * 4^(3-g), an unsigned byte.  One dp4a per group,
// word and token accumulates sum code*x scaled by 4^(3-g) in its own
// register; the four are rescaled exactly (arithmetic shifts of exact
// multiples) and summed at the end of the tile, and sum_k x is subtracted
// because w = code - 1.  Bytes of a box past K read as zero, i.e. code 0,
// and contribute nothing.
#pragma once

#include "ptx.cuh"
#include "quant_kernels.cuh"

namespace bitnet {

constexpr int kGemvTileRows = 128;
constexpr int kGemvMaxK = 8192;      // the x slot holds M x K bytes, K <= 8192 ...
constexpr int kGemvMaxKLong = 30720;  // ... or, in the one-token long-K variant, K <= 30720

// One independent problem of a batch (device pointers and shape).
//
// Split K: a problem with few row tiles can have its K range cut into
// `splits` slices of `cps` boxes each; a work item is then one (slice, row
// tile) pair, numbered slice by slice.  Each item adds up its slice into
// int32 partial sums in the workspace; the last of the slices of a row tile
// to finish (per warp, counted in the workspace) adds the partials in slice
// order and writes the outputs.  Integer sums are exact, so the results are
// the same as without the split.
struct BatchProblem {
  const uint8_t* packed;  // I2_S tensor [n, k]
  int8_t* xq;             // int8 activations [m, k]
  float* xs;              // per-token scales [m]
  float* y;               // [m, n]
  int32_t* acc;           // [m, n] or null
  int32_t n, k;
  int32_t item_start;     // first global work item of this problem
  int32_t stage_start;    // first global stage (one box each) of this problem
  int32_t splits;         // K slices (1: no split)
  int32_t cps;            // boxes per slice (the last slice may have fewer)
  int32_t part_off;       // partial sums: split_base + part_off, [tile][slice][MT][128]
  int32_t cnt_off;        // arrival counters: cnt_base + cnt_off, [tile][4 warps]
};

template <int CAP>
struct BatchParamsT {
  int32_t count;         // problems
  int32_t m;             // tokens (the same for every problem)
  int32_t total_items;   // row tiles over all problems
  int32_t total_stages;  // boxes over all problems
  int32_t pdl;           // 1: activations come from the preceding grid
  int32_t dyn_start;     // items from here on are handed out through `queue`
  int32_t* queue;        // zeroed work counter, or null: every item in a fixed range
  int32_t static_stages; // stages of the items before dyn_start
  int32_t pad;
  int32_t* split_base;   // partial sums of split problems (workspace), or null
  int32_t* cnt_base;     // their zeroed arrival counters (workspace), or null
  CUtensorMap tmap[CAP];  // per problem: packed bytes as [n rows, k/4 bytes], box 128 x 128
  BatchProblem p[CAP];
};

struct StageMeta {
  int32_t p;     // problem
  int32_t row0;  // first row of the tile
  int32_t kc;    // box index along K (512 weights each)
  int32_t info;  // bit 0: first box of the tile, bit 1: last box, bits 8..: switch index + 1
};

template <int MT, int KMAX = kGemvMaxK>
struct GemvCfg {
  static_assert(MT >= 1 && MT <= 2, "tokens");
  static_assert(KMAX == kGemvMaxK || (MT == 1 && KMAX == kGemvMaxKLong), "variant");
  static constexpr int kComputeWarps = kGemvTileRows / 32;
  static constexpr int kThreads = 32 * (kComputeWarps + 1);
  static constexpr int kBoxBytes = kGemvTileRows * 128;  // 16 KB
  // One token: 3 stages and 3 CTAs per SM (2 with the long-K activation
  // slots); two tokens: 4 stages, 2 CTAs.
  static constexpr int kStages = MT == 1 ? 3 : 4;
  static constexpr int kCtasPerSm = (MT == 1 && KMAX == kGemvMaxK) ? 3 : 2;
  static constexpr int kXSlotBytes = MT * KMAX + 512;  // + slack read past K, never used
  static constexpr int kBars = 2 * kStages + 4;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kBoxBytes +
                                       2 * kXSlotBytes + kBars * 8 +
                                       kStages * sizeof(StageMeta) + 2 * 4 * sizeof(float) + 16;
};

__device__ __forceinline__ int dp4a_u8s8(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

template <typename BP>
__device__ __forceinline__ int find_problem_by_item(const BP& bp, int item) {
  int lo = 0, hi = bp.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (bp.p[mid].item_start <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// First item whose first stage is at or after global stage `target`; the
// items of one problem are counted as `cps` stages each.
template <typename BP>
__device__ __forceinline__ int first_item_at_stage(const BP& bp, int target) {
  if (target >= bp.total_stages) return bp.total_items;
  int lo = 0, hi = bp.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (bp.p[mid].stage_start <= target) lo = mid;
    else hi = mid - 1;
  }
  const BatchProblem& P = bp.p[lo];
  const int nk = P.cps;
  const int items = ((P.n + kGemvTileRows - 1) / kGemvTileRows) * P.splits;
  const int off = (target - P.stage_start + nk - 1) / nk;
  return off >= items ? P.item_start + items : P.item_start + off;
}

// Row tile, slice and box range [kc_lo, kc_hi) of item `item` of problem P.
__device__ __forceinline__ void split_item(const BatchProblem& P, int item, int* rt, int* sl,
                                           int* kc_lo, int* kc_hi) {
  const int tiles = (P.n + kGemvTileRows - 1) / kGemvTileRows;
  const int local = item - P.item_start;
  *sl = local / tiles;
  *rt = local - *sl * tiles;
  *kc_lo = *sl * P.cps;
  *kc_hi = min((P.k + 511) >> 9, *kc_lo + P.cps);
}

template <int MT, int CAP, int KMAX = kGemvMaxK>
__global__ void __launch_bounds__(GemvCfg<MT, KMAX>::kThreads, GemvCfg<MT, KMAX>::kCtasPerSm)
    i2s_gemv_dp4a_kernel(const __grid_constant__ BatchParamsT<CAP> bp) {
  using C = GemvCfg<MT, KMAX>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* boxes = smem;
  uint8_t* xslots = smem + S * C::kBoxBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(xslots + 2 * C::kXSlotBytes);
  StageMeta* meta = reinterpret_cast<StageMeta*>(bars + C::kBars);
  float* xscal = reinterpret_cast<float*>(meta + S);  // per slot: weight scale, xs[0..MT)
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

  const int m_tokens = bp.m;
  // Fixed ranges over the items before dyn_start, balanced by stages.
  const int64_t ts = bp.static_stages;
  const int item_lo = first_item_at_stage(bp, static_cast<int>(ts * blockIdx.x / gridDim.x));
  const int item_hi = first_item_at_stage(bp, static_cast<int>(ts * (blockIdx.x + 1) / gridDim.x));

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane != 0) {
      if (bp.pdl) grid_dependency_wait();
      grid_dependents_launch();
    } else {
      int issued = 0;    // boxes issued
      int nsw = 0;       // problem switches announced to the consumers
      int x_loaded = 0;  // switches whose activations were requested
      int prev_p = -1, prev_sl = -1;
      bool waited = (bp.pdl == 0);
      if (waited) grid_dependents_launch();
      // Items: first this CTA's fixed range, then, with a work queue, items
      // from dyn_start on, one at a time, as the CTA becomes free (the counter
      // is zeroed by the preceding grid, so it is read only after the wait).
      // The fixed ranges keep every CTA on neighbouring tiles of one problem
      // for most of the launch; the shared tail evens out the finishing times.
      const bool dyn = bp.queue != nullptr;
      int next = 0;
      bool have_next = false;
      auto grab = [&]() {  // its result is used one item later
        next = bp.dyn_start + atomicAdd(bp.queue, 1);
        have_next = true;
      };
      // The weights do not depend on the preceding grid: the first stages are
      // issued before waiting for it.
      auto wait_for_inputs = [&]() {
        grid_dependency_wait();
        grid_dependents_launch();
        waited = true;
      };
      // Weights are read once: they go first when L2 needs room, so that the
      // activations the next CTAs read stay there.
      const uint64_t pol_w = l2_policy_evict_first();
      int sw_problem[2] = {-1, -1};  // problem of each switch not yet loaded
      int sw_klo[2] = {0, 0};        // first activation of its slot (K slices)
      bool ok = true;
      // Request the activations (and scales) of switch `j` into slot j & 1.
      auto load_x = [&](int j) -> bool {
        const int slot = j & 1;
        if (j >= 2 && !mbar_wait(xempty_bar(slot), ((j >> 1) - 1) & 1, abort_flag)) return false;
        const BatchProblem& P = bp.p[sw_problem[slot]];
        xscal[4 * slot] =
            *reinterpret_cast<const float*>(P.packed + static_cast<size_t>(P.n) * (P.k >> 2));
#pragma unroll
        for (int m = 0; m < MT; ++m) xscal[4 * slot + 1 + m] = (m < m_tokens) ? P.xs[m] : 0.0f;
        if (P.k <= KMAX) {
          const uint32_t xbytes = static_cast<uint32_t>(m_tokens) * static_cast<uint32_t>(P.k);
          mbar_arrive_expect_tx(xfull_bar(slot), xbytes);  // publishes xscal[slot]
          bulk_load(smem_u32(xslots + slot * C::kXSlotBytes), P.xq, xbytes, xfull_bar(slot));
        } else {
          // A K slice: each token's activations k_lo .. k_hi, one after the other.
          const int k_lo = sw_klo[slot];
          const uint32_t len = static_cast<uint32_t>(min(P.k, k_lo + P.cps * 512) - k_lo);
          mbar_arrive_expect_tx(xfull_bar(slot), static_cast<uint32_t>(m_tokens) * len);
          for (int m = 0; m < m_tokens; ++m)
            bulk_load(smem_u32(xslots + slot * C::kXSlotBytes + m * len),
                      P.xq + static_cast<int64_t>(m) * P.k + k_lo, len, xfull_bar(slot));
        }
        return true;
      };
      auto load_pending_x = [&]() {
        while (ok && x_loaded < nsw) {
          ok = load_x(x_loaded);
          ++x_loaded;
        }
      };
      int item = item_lo;
      bool in_static = item_lo < item_hi;
      if (!in_static) {
        if (dyn) {
          if (!waited) wait_for_inputs();
          grab();
          item = next;
          have_next = false;
        } else {
          item = bp.total_items;
        }
      }
      while (ok && item < bp.total_items) {
        // The next shared item is requested while the last fixed one (or a
        // shared one) is issued, so the atomic's round trip is hidden.
        if (dyn && waited && !have_next && (!in_static || item + 1 >= item_hi)) grab();
        const int p = find_problem_by_item(bp, item);
        const BatchProblem& P = bp.p[p];
        int rt, sl, kc_lo, kc_hi;
        split_item(P, item, &rt, &sl, &kc_lo, &kc_hi);
        const int row0 = rt * kGemvTileRows;
        for (int kc = kc_lo; kc < kc_hi; ++kc) {
          const int s = issued % S;
          if (issued >= S) {
            if (!waited) {
              // Activations and scales come from the preceding grid.
              wait_for_inputs();
              load_pending_x();
              if (!ok) break;
            }
            if (!mbar_wait(empty_bar(s), ((issued / S) - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
          }
          int info = (kc == kc_lo ? 1 : 0) | (kc == kc_hi - 1 ? 2 : 0);
          // A new problem, or a new K slice of one too long for the slot.
          if (kc == kc_lo && (p != prev_p || (P.k > KMAX && sl != prev_sl))) {
            // At most two switches wait for their activations: the slots.
            if (nsw - x_loaded >= 2) {
              if (!waited) wait_for_inputs();
              load_pending_x();
              if (!ok) break;
            }
            prefetch_tensormap(&bp.tmap[p]);
            sw_problem[nsw & 1] = p;
            sw_klo[nsw & 1] = P.k > KMAX ? kc_lo * 512 : 0;
            info |= (nsw + 1) << 8;
            ++nsw;
            prev_p = p;
            prev_sl = sl;
          }
          StageMeta md;
          md.p = p;
          md.row0 = row0;
          md.kc = kc;
          md.info = info;
          meta[s] = md;
          mbar_arrive_expect_tx(full_bar(s), C::kBoxBytes);  // publishes meta[s]
          tma_load_2d_hint(smem_u32(boxes + s * C::kBoxBytes), &bp.tmap[p], kc * 128, row0,
                           full_bar(s), pol_w);
          ++issued;
          if (waited) load_pending_x();
        }
        if (!ok) break;
        if (in_static && item + 1 < item_hi) {
          ++item;
        } else if (dyn) {
          if (!have_next) {
            if (!waited) {
              // Activations whose loads waited for the preceding grid go
              // out now: the next box may need a stage that the compute
              // warps free only once they have them.
              wait_for_inputs();
              load_pending_x();
              if (!ok) break;
            }
            grab();
          }
          item = next;
          have_next = false;
          in_static = false;
        } else {
          break;
        }
      }
      if (!waited) wait_for_inputs();
      load_pending_x();
      if (ok) {
        // End of the work: a stage without data whose meta says so.
        const int s = issued % S;
        if (issued < S || mbar_wait(empty_bar(s), ((issued / S) - 1) & 1, abort_flag)) {
          StageMeta md;
          md.p = -1;
          md.row0 = 0;
          md.kc = 0;
          md.info = 0;
          meta[s] = md;
          mbar_arrive(full_bar(s));  // publishes meta[s]
        }
      }
      // This CTA does not finish before the preceding grid has, so that the
      // completion of any grid in a chain implies that of all before it.
      grid_dependency_wait();
      if (*abort_flag) {
        // Let the copies still in flight land before shared memory goes away.
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait(full_bar(i % S), (i / S) & 1, nullptr, kDrainTimeoutNs);
        for (int j = (x_loaded > 2 ? x_loaded - 2 : 0); j < x_loaded; ++j)
          mbar_wait(xfull_bar(j & 1), (j >> 1) & 1, nullptr, kDrainTimeoutNs);
      }
    }
    return;
  }

  // ---------------------------------------------------------------- compute
  const int cw = warp - 1;
  const int rs = lane >> 2;  // row slot: rows 32*cw + rs + 8*i of the tile
  const int cp = lane & 3;   // I2_S block of the box this lane reads
  // Visit order of the groups for this lane: j -> group (j + cp) % 4.
  uint32_t gmask[4];
  int gshift[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int g = (j + cp) & 3;
    gshift[j] = 6 - 2 * g;
    gmask[j] = 0x03030303u << gshift[j];
  }
  if (bp.pdl) grid_dependency_wait();
  grid_dependents_launch();
  int a[4][MT][4];  // [row i][token][visit j]: sum of code_g * x * 4^(3-g), g = (j + cp) % 4
  int xsum[MT];
  float xsv[MT];
  float wscale = 0.0f;
  const uint8_t* xsm = xslots;
  int cur_slot = -1;
  int k = 0, n = 0, splits = 1;
  int xoff = 0, xstride = 0;  // the slot holds activations xoff .. xoff + xstride of each token
  int kc_first = 0;  // first box of the current item
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    xsum[m] = 0;
    xsv[m] = 0.0f;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int g = 0; g < 4; ++g) a[i][m][g] = 0;
  int s = 0;
  uint32_t phase = 0;
  while (true) {
    if (!__all_sync(0xffffffffu, mbar_wait(full_bar(s), phase, abort_flag))) break;
    StageMeta md;
    {
      const volatile int32_t* vm = reinterpret_cast<const volatile int32_t*>(meta + s);
      md.p = vm[0];
      md.row0 = vm[1];
      md.kc = vm[2];
      md.info = vm[3];
    }
    if (md.p < 0) break;  // the producer has no more work
    const int sw = (md.info >> 8) - 1;
    if (sw >= 0) {
      // A new problem: release the previous slot, take the new one.
      if (cur_slot >= 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(xempty_bar(cur_slot));
      }
      const int slot = sw & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(xfull_bar(slot), (sw >> 1) & 1, abort_flag))) break;
      cur_slot = slot;
      xsm = xslots + slot * C::kXSlotBytes;
      k = bp.p[md.p].k;
      n = bp.p[md.p].n;
      splits = bp.p[md.p].splits;
      xoff = k > KMAX ? md.kc * 512 : 0;
      xstride = k > KMAX ? min(k, xoff + bp.p[md.p].cps * 512) - xoff : k;
      wscale = xscal[4 * slot];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        xsv[m] = xscal[4 * slot + 1 + m];
        int sum = 0;
        if (m < m_tokens && splits == 1) {
          for (int off = lane * 16; off < k; off += 512) {
            const uint4 v = *reinterpret_cast<const uint4*>(xsm + m * xstride + off);
            sum = __dp4a(static_cast<int>(v.x), 0x01010101, sum);
            sum = __dp4a(static_cast<int>(v.y), 0x01010101, sum);
            sum = __dp4a(static_cast<int>(v.z), 0x01010101, sum);
            sum = __dp4a(static_cast<int>(v.w), 0x01010101, sum);
          }
        }
        xsum[m] = __reduce_add_sync(0xffffffffu, sum);
      }
    }
    if (md.info & 1) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int g = 0; g < 4; ++g) a[i][m][g] = 0;
      kc_first = md.kc;
      if (splits > 1) {
        // A slice of K: sum_k x over the slice's range only.
        const int k_lo = md.kc * 512;
        const int k_hi = min(k, k_lo + bp.p[md.p].cps * 512);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          int sum = 0;
          if (m < m_tokens) {
            for (int off = k_lo + lane * 16; off < k_hi; off += 512) {
              const uint4 v = *reinterpret_cast<const uint4*>(xsm + m * xstride + (off - xoff));
              sum = __dp4a(static_cast<int>(v.x), 0x01010101, sum);
              sum = __dp4a(static_cast<int>(v.y), 0x01010101, sum);
              sum = __dp4a(static_cast<int>(v.z), 0x01010101, sum);
              sum = __dp4a(static_cast<int>(v.w), 0x01010101, sum);
            }
          }
          xsum[m] = __reduce_add_sync(0xffffffffu, sum);
        }
      }
    }
    const int kblk = md.kc * 512 + 128 * cp;  // first weight of this lane's block
    if (kblk < k) {                            // blocks wholly past K are skipped
      // Activations of the block: group g, words 0..7 = k = kblk + 32g + 0..31,
      // in this lane's visit order.
      uint32_t xr[MT][4][8];
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint8_t* xg = xsm + m * xstride + (kblk - xoff) + 32 * ((j + cp) & 3);
          const uint4 lo = *reinterpret_cast<const uint4*>(xg);
          const uint4 hi = *reinterpret_cast<const uint4*>(xg + 16);
          xr[m][j][0] = lo.x;
          xr[m][j][1] = lo.y;
          xr[m][j][2] = lo.z;
          xr[m][j][3] = lo.w;
          xr[m][j][4] = hi.x;
          xr[m][j][5] = hi.y;
          xr[m][j][6] = hi.z;
          xr[m][j][7] = hi.w;
        }
      const uint8_t* box = boxes + s * C::kBoxBytes;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = cw * 32 + rs + 8 * i;  // row of the tile; r & 7 == rs
        const uint8_t* wrow = box + r * 128;
        const uint4 w0 = *reinterpret_cast<const uint4*>(wrow + (((2 * cp) ^ rs) << 4));
        const uint4 w1 = *reinterpret_cast<const uint4*>(wrow + (((2 * cp + 1) ^ rs) << 4));
        const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        // Visit order: with two tokens, consecutive dp4a feed different
        // accumulators (word-major), which measured about 3 % faster; one
        // token keeps group-major order.
#pragma unroll
        for (int o = 0; o < 32; ++o) {
          const int j = MT == 1 ? o / 8 : o % 4;
          const int q = MT == 1 ? o % 8 : o / 4;
          const uint32_t v = wv[q] & gmask[j];
#pragma unroll
          for (int m = 0; m < MT; ++m) a[i][m][j] = dp4a_u8s8(v, xr[m][j][q], a[i][m][j]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
    if (++s == S) {
      s = 0;
      phase ^= 1u;
    }
    if (md.info & 2) {
      // Tile done: add the 4 block lanes of each row, then
      // y = ((float)acc * xs[m]) * s.
      const BatchProblem& P = bp.p[md.p];
      if (splits == 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t row = static_cast<int64_t>(md.row0) + cw * 32 + rs + 8 * i;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            int part = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) part += a[i][m][j] >> gshift[j];
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (cp == 0 && m < m_tokens && row < n) {
              const int dot = part - xsum[m];
              P.y[m * static_cast<int64_t>(n) + row] =
                  __fmul_rn(__fmul_rn(__int2float_rn(dot), xsv[m]), wscale);
              if (P.acc != nullptr) P.acc[m * static_cast<int64_t>(n) + row] = dot;
            }
          }
        }
      } else {
        // One slice of a split problem: this warp's 32 rows of partial sums
        // go to the workspace; the warp that brings the last slice of these
        // rows adds all slices (in slice order) and writes the outputs.
        const int rt = md.row0 / kGemvTileRows;
        const int sl = kc_first / P.cps;
        int32_t* tile_part =
            bp.split_base + P.part_off + static_cast<int64_t>(rt) * splits * (MT * 128);
        int32_t* mine = tile_part + static_cast<int64_t>(sl) * (MT * 128);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            int part = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) part += a[i][m][j] >> gshift[j];
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (cp == 0 && m < m_tokens) mine[m * 128 + cw * 32 + rs + 8 * i] = part - xsum[m];
          }
        }
        __threadfence();
        __syncwarp();
        int32_t* cnt = bp.cnt_base + P.cnt_off + rt * 4 + cw;
        int last = 0;
        if (lane == 0) last = atomicAdd(cnt, 1) == splits - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          const int64_t row = static_cast<int64_t>(md.row0) + cw * 32 + lane;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m < m_tokens) {
              int dot = 0;
              for (int q = 0; q < splits; ++q)
                dot += __ldcg(tile_part + q * (MT * 128) + m * 128 + cw * 32 + lane);
              if (row < n) {
                P.y[m * static_cast<int64_t>(n) + row] =
                    __fmul_rn(__fmul_rn(__int2float_rn(dot), xsv[m]), wscale);
                if (P.acc != nullptr) P.acc[m * static_cast<int64_t>(n) + row] = dot;
              }
            }
          }
          if (lane == 0) *cnt = 0;  // ready for the next call on this workspace
        }
      }
    }
  }
}

// Zeroes the work counters of the decode launches that follow, once the
// preceding grid (and with it every earlier user of the counters) is done.
__global__ void __launch_bounds__(256) zero_counters_kernel(int32_t* queue, int32_t n) {
  grid_dependency_wait();
  for (int i = threadIdx.x; i < n; i += blockDim.x) queue[i] = 0;
  grid_dependents_launch();
}

// Per-token absmax quantization of many problems' activations in one launch:
// one CTA per (problem, token) row, the same arithmetic as act_quant_kernel.
constexpr int kQuantBatch = 1000;

struct QuantProblem {
  const float* x;  // [m, k] fp32
  int8_t* xq;      // [m, k] int8
  float* xs;       // [m]
  int64_t k;
};

struct QuantBatchParams {
  int32_t count;
  int32_t m;
  int32_t* queue;  // work counters of the decode launches that follow, zeroed here (or null)
  int32_t nqueue;
  int32_t pad;
  QuantProblem p[kQuantBatch];
};

__global__ void __launch_bounds__(256) act_quant_batched_kernel(
    const __grid_constant__ QuantBatchParams qp) {
  grid_dependency_wait();
  grid_dependents_launch();
  // The preceding grid (and so every earlier user of the counters) is done.
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < qp.nqueue; i += blockDim.x) qp.queue[i] = 0;
  __shared__ float red[32];
  const int p = blockIdx.x / qp.m;
  const int m = blockIdx.x % qp.m;
  const QuantProblem& P = qp.p[p];
  quantize_row(P.x + static_cast<int64_t>(m) * P.k, P.k, P.xq + static_cast<int64_t>(m) * P.k,
               P.xs + m, red);
}

}  // namespace bitnet
