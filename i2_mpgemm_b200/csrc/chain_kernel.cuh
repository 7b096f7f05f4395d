// chain_kernel.cuh -- a dependency-ordered sequence of fused quantize + I2_S
// matmul problems (one or two tokens) in one persistent launch.
//
// A BitNet b1.58 layer has seven ternary projections, q, k, v, o, gate, up
// and down ("BitNet Inference Preprocessing: Converting Hugging Face
// Checkpoints to I2S GGUF", The Two-Stage BitNet Inference Preprocessing
// Pipeline), and each quantizes its input per token with absmax to int8
// before the ternary contraction ("LLM Quantization Paradigms: FP8, AWQ,
// EXL2 & BitNet b1.58 in 2026", section 5).  In a decode step they form a
// chain: q, k and v read the layer input, o reads the attention output, gate
// and up read o's, down reads the FFN's, and down's output feeds the next
// layer.  Run as separate calls, every link costs a grid completion and a
// relaunch, far more than the 0.3-1.4 us its weights take to stream.  Here
// the whole chain is one launch:
//
//   * A problem's input is either an external fp32 tensor or the output of
//     one earlier problem (its `src`).  Problems come in dependency order.
//   * Work item = (problem, K slice, row tile), numbered problem by problem;
//     item i belongs to CTA i mod grid, and each CTA works through its items
//     in increasing order.  A stage has at most about as many items as the
//     grid has CTAs, so its items run on different CTAs side by side.  The
//     producer warp streams the items' weight boxes (TMA, evict-first) into
//     a ring: the weights do not depend on anything, so the ring fills with
//     the CTA's next items' weights while the compute warps wait for an
//     earlier item's input.
//   * Item start: the compute warps read the source problem's whole output,
//     each 128-row tile as soon as its counter in the workspace says all of
//     its K slices are in (bounded waits), take the token's absmax over it,
//     and quantize just the item's K slice into shared memory.  The source's outputs are
//     read as its exact int32 accumulators and turned into fp32 with the
//     source's own scales, y = ((float)acc * xs) * s, the same operations
//     and order as the output it writes, so every quantized value is the one
//     a separate call would compute from that output.  Because |y| is a
//     non-decreasing function of |acc| (int -> float and multiplication by a
//     non-negative scale round monotonically, and symmetrically in sign),
//     the absmax of the output is y(max |acc|), exactly.
//   * Item end: the slice's int32 row sums go to the problem's accumulators
//     in the workspace (a plain store when the problem has one slice, an
//     atomic add otherwise: integer sums are exact in any order); then one
//     release add counts the slice in its row tile's counter.  The CTA that
//     brings the last slice of a row tile writes the tile's fp32 outputs (and
//     the optional int32 copy) for the caller.
//
// Progress: an item waits only for items of earlier problems, which have
// lower numbers; each CTA works through its items in increasing order, and
// the launch is cooperative, so every CTA is resident.  So the lowest
// unfinished item never waits on anything unfinished, and the chain always
// advances.  Every wait is bounded all the same (device error flag, CTA
// abort).
//
// The per-box arithmetic is the decode kernel's: mask-without-shift dp4a on
// the 128-byte-swizzled box, four lanes per row, one I2_S block per lane.
#pragma once

#include "gemv_kernel.cuh"

namespace bitnet {

constexpr int kChainMaxCps = 16;  // boxes per item at most: 8192 activations per token
constexpr int kChainBatch = 128;  // problems per launch (parameter block under 32 KB)
// One-token chains also count finished items per problem; these counters sit
// 256 bytes apart, since all CTAs of a stage poll one of them at once.
constexpr int kChainDoneStride = 64;

struct ChainProblem {
  const uint8_t* packed;   // I2_S tensor [n, k]
  const float* x;          // external input [m, k] fp32 (src < 0)
  const float* src_scale;  // weight scale of the source problem (src >= 0)
  float* y;                // [m, n]
  int32_t* acc_out;        // [m, n] or null
  int32_t n, k;
  int32_t idx;        // index in the whole chain: scale slot and done counter
  int32_t src;        // chain index of the problem whose output is the input, or -1
  int32_t src_splits; // that problem's K slices: a row tile of it is complete at this count
  int32_t src_items;  // that problem's work items (all done: its output is complete)
  int32_t src_cnt;    // its row-tile counters: cnt_base + src_cnt, [k / 128]
  int32_t src_acc;    // its accumulators: acc_base + src_acc, [m][k]
  int32_t acc;        // this problem's accumulators: acc_base + acc, [m][n]
  int32_t cnt;        // its row-tile arrival counters: cnt_base + cnt, [tiles]
  int32_t item_start; // first work item of this problem in its launch
  int32_t splits;     // K slices
  int32_t cps;        // boxes per slice (the last slice may have fewer)
};

template <int CAP>
struct ChainParamsT {
  int32_t count;        // problems in this launch
  int32_t m;            // tokens
  int32_t total_items;  // work items of this launch
  int32_t pad;
  int32_t* done;        // per chain problem, kChainDoneStride ints apart: finished items (zeroed)
  int32_t* cnt_base;    // per row tile: finished slices (zeroed)
  int32_t* acc_base;    // int32 accumulators (zeroed)
  float* xs_base;       // per chain problem: two activation scales
  CUtensorMap tmap[CAP];  // per problem: packed bytes as [n rows, k/4 bytes], box 128 x 128
  ChainProblem p[CAP];
};

template <int MT>
struct ChainCfg {
  static_assert(MT >= 1 && MT <= 2, "tokens");
  static constexpr int kComputeWarps = 4;
  static constexpr int kThreads = 32 * (kComputeWarps + 1);
  static constexpr int kBoxBytes = kGemvTileRows * 128;
  static constexpr int kStages = MT == 1 ? 3 : 4;
  static constexpr int kCtasPerSm = MT == 1 ? 3 : 2;
  static constexpr int kXBytes = MT * kChainMaxCps * 512;
  static constexpr int kBars = 2 * kStages + 1;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kBoxBytes + kXBytes +
                                       kBars * 8 + kStages * sizeof(StageMeta) + 128;
};

__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_gpu_add(int32_t* p, int32_t v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int32_t atom_acq_rel_gpu_add(int32_t* p, int32_t v) {
  int32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Bounded wait until *ctr >= target (acquire loads at gpu scope).  Gives
// up when `abort` is raised by another thread of the CTA, or after
// kWaitTimeoutNs, raising `abort` and the device error flag.  Polls are
// 32 ns apart.  (Measured: a longer or growing back-off, several staggered
// pollers per CTA, or relaxed polls plus a fence change nothing or cost
// time.)
__device__ __forceinline__ bool wait_count(const int32_t* ctr, int32_t target,
                                           volatile uint32_t* abort) {
  const uint64_t t0 = global_timer_ns();
  for (int i = 0;; ++i) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    __nanosleep(32);
    if ((i & 15) == 15) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > kWaitTimeoutNs) {
        *abort = 1u;
        atomicOr(&g_error_flags, kErrWaitTimeout);
        return false;
      }
    }
  }
}

template <int CAP>
__device__ __forceinline__ int chain_problem_of(const ChainParamsT<CAP>& cp, int item) {
  int lo = 0, hi = cp.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cp.p[mid].item_start <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

template <int MT, int CAP>
__global__ void __launch_bounds__(ChainCfg<MT>::kThreads, ChainCfg<MT>::kCtasPerSm)
    i2s_chain_kernel(const __grid_constant__ ChainParamsT<CAP> cp) {
  using C = ChainCfg<MT>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* boxes = smem;
  uint8_t* xbuf = smem + S * C::kBoxBytes;  // [MT][cps * 512] int8 of the current item
  uint64_t* bars = reinterpret_cast<uint64_t*>(xbuf + C::kXBytes);
  StageMeta* meta = reinterpret_cast<StageMeta*>(bars + C::kBars);
  uint32_t* red = reinterpret_cast<uint32_t*>(meta + S);  // [0,8): maxima, [8,16): sums
  volatile uint32_t* abort_flag = red + 16;
  volatile uint32_t* last_flag = red + 17;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t cbar = bar0 + 8u * (2 * S);  // the compute warps' own barrier

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), C::kComputeWarps);
    }
    mbar_init(cbar, C::kComputeWarps);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The zeroed counters, and every input, come from earlier grids.
    grid_dependency_wait();
    grid_dependents_launch();
    if (lane != 0) return;
    const uint64_t pol_w = l2_policy_evict_first();
    int issued = 0;
    bool ok = true;
    // Item i belongs to CTA i mod grid (the launch is cooperative: every
    // CTA is resident), so the items of one stage run on different CTAs,
    // side by side, and each CTA takes its items in increasing order.
    for (int item = blockIdx.x; ok && item < cp.total_items; item += gridDim.x) {
      const int p = chain_problem_of(cp, item);
      const ChainProblem& P = cp.p[p];
      const int tiles = (P.n + kGemvTileRows - 1) / kGemvTileRows;
      const int local = item - P.item_start;
      const int sl = local / tiles;
      const int row0 = (local - sl * tiles) * kGemvTileRows;
      const int kc_lo = sl * P.cps;
      const int kc_hi = min((P.k + 511) >> 9, kc_lo + P.cps);
      prefetch_tensormap(&cp.tmap[p]);
      for (int kc = kc_lo; kc < kc_hi; ++kc) {
        const int s = issued % S;
        if (issued >= S && !mbar_wait(empty_bar(s), ((issued / S) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        StageMeta md;
        md.p = p;
        md.row0 = row0;
        md.kc = kc;
        md.info = (kc == kc_lo ? 1 : 0) | (kc == kc_hi - 1 ? 2 : 0);
        meta[s] = md;
        mbar_arrive_expect_tx(full_bar(s), C::kBoxBytes);  // publishes meta[s]
        tma_load_2d_hint(smem_u32(boxes + s * C::kBoxBytes), &cp.tmap[p], kc * 128, row0,
                         full_bar(s), pol_w);
        ++issued;
      }
    }
    ok = ok && *abort_flag == 0u;
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
    if (*abort_flag) {
      // Let the copies still in flight land before shared memory goes away.
      for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
        mbar_wait(full_bar(i % S), (i / S) & 1, nullptr, kDrainTimeoutNs);
    }
    return;
  }

  // ---------------------------------------------------------------- compute
  grid_dependency_wait();
  grid_dependents_launch();
  const int cw = warp - 1;
  const int ctid = threadIdx.x - 32;
  const int rs = lane >> 2;  // row slot: rows 32*cw + rs + 8*i of the tile
  const int cq = lane & 3;   // I2_S block of the box this lane reads
  uint32_t gmask[4];
  int gshift[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int g = (j + cq) & 3;
    gshift[j] = 6 - 2 * g;
    gmask[j] = 0x03030303u << gshift[j];
  }
  uint32_t cphase = 0;
  // All four compute warps meet; false when the CTA is aborting.  The
  // second __syncwarp keeps the other lanes from probing the barrier before
  // lane 0 has arrived: a diverged warp could otherwise spin on a phase that
  // only its own lane 0, not yet scheduled, can complete.
  auto csync = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    __syncwarp();
    const bool ok = mbar_wait_spin(cbar, cphase, abort_flag);
    cphase ^= 1u;
    return __all_sync(0xffffffffu, ok) && *abort_flag == 0u;
  };

  int a[4][MT][4];
  int xsum[MT];
  float xsp[MT];   // activation scale of the current problem
  float wscale = 0.0f;
  int xoff = 0, xstride = 0;
  // Absmax of the last input seen (source problem or external pointer).
  int cached_src = -2, cached_k = 0;
  const float* cached_x = nullptr;
  float amax[MT];
  float xs_in[MT];  // activation scales of the source problem
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    xsum[m] = 0;
    xsp[m] = 0.0f;
    amax[m] = 0.0f;
    xs_in[m] = 0.0f;
  }
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
    const ChainProblem& P = cp.p[md.p];
    if (md.info & 1) {
      // ------------------------------------------------ item start
      // Nobody reads the previous item's activations any more.
      if (!csync()) break;
      const int k = P.k;
      const int k_lo = md.kc * 512;
      const int k_hi = min(k, k_lo + P.cps * 512);
      const int nr = (k_hi - k_lo + 511) >> 9;  // 512-weight chunks in the slice
      xoff = k_lo;
      xstride = nr * 512;
      wscale = __ldg(reinterpret_cast<const float*>(P.packed + static_cast<size_t>(P.n) * (k >> 2)));
      const bool chained = P.src >= 0;
      const float s_src = chained ? __ldg(P.src_scale) : 0.0f;
      const bool fresh = chained ? cached_src != P.src
                                 : (cached_src != -1 || cached_x != P.x || cached_k != k);
      // The input row, as int4 words (int32 accumulators, or fp32 bits):
      // thread ctid owns elements 4*ctid .. 4*ctid+3 of every 512-chunk.
      const int4* src4 = chained ? reinterpret_cast<const int4*>(cp.acc_base + P.src_acc)
                                 : reinterpret_cast<const int4*>(P.x);
      // This thread's words of the slice's first two chunks, kept from the
      // absmax pass so that slices of one or two chunks need no second read.
      int4 keep[MT][2];
      const bool kept = nr <= 2;
      if (fresh && MT == 1) {
        // One token: wait until every item of the source is done (one poller
        // per CTA on the source's done counter), then read the whole row,
        // eight 512-chunks per batch with their loads in flight together.
        // The CTAs of a stage all read the same row at once; each starts at
        // its own chunk, so that they do not sweep its lines in step.
        if (chained && ctid == 0)
          wait_count(cp.done + P.src * kChainDoneStride, P.src_items, abort_flag);
        if (!csync()) break;
        if (chained && ctid < MT)
          red[20 + ctid] = __float_as_uint(__ldcg(cp.xs_base + 2 * P.src + ctid));
        constexpr int kB = 8;
        const int nch = (k + 511) >> 9;
        const int rot = static_cast<int>(blockIdx.x % static_cast<unsigned>(nch));
        uint32_t mx = 0;
        keep[0][0] = make_int4(0, 0, 0, 0);
        keep[0][1] = make_int4(0, 0, 0, 0);
        for (int t0 = 0; t0 < nch; t0 += kB) {
          int4 vb[kB];
          int rr[kB];
#pragma unroll
          for (int u = 0; u < kB; ++u) {
            const int r = t0 + u + rot < nch ? t0 + u + rot : t0 + u + rot - nch;
            rr[u] = t0 + u < nch && r * 512 + 4 * ctid < k ? r : -1;
            vb[u] = rr[u] >= 0 ? src4[rr[u] * 128 + ctid] : make_int4(0, 0, 0, 0);
          }
#pragma unroll
          for (int u = 0; u < kB; ++u) {
            const int4 v = vb[u];
            if (rr[u] == md.kc) keep[0][0] = v;
            if (rr[u] >= 0 && rr[u] == md.kc + 1) keep[0][1] = v;
            if (chained) {
              mx = max(mx, max(max(static_cast<uint32_t>(abs(v.x)), static_cast<uint32_t>(abs(v.y))),
                               max(static_cast<uint32_t>(abs(v.z)), static_cast<uint32_t>(abs(v.w)))));
            } else {
              // Non-negative floats order like their bit patterns.
              mx = max(mx, max(max(static_cast<uint32_t>(v.x) & 0x7fffffffu,
                                   static_cast<uint32_t>(v.y) & 0x7fffffffu),
                               max(static_cast<uint32_t>(v.z) & 0x7fffffffu,
                                   static_cast<uint32_t>(v.w) & 0x7fffffffu)));
            }
          }
        }
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (lane == 0) red[cw * 2] = mx;
        if (!csync()) break;
        if (chained) xs_in[0] = __uint_as_float(red[20]);
        const uint32_t m0 = max(max(red[0], red[2]), max(red[4], red[6]));
        amax[0] = chained ? __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(m0)), xs_in[0]), s_src)
                          : __uint_as_float(m0);
        cached_src = chained ? P.src : -1;
        cached_x = chained ? nullptr : P.x;
        cached_k = k;
      } else if (fresh) {
        // Two tokens: stream the source row in as its row tiles complete.  Chunk r (512
        // values) holds row tiles 4r .. 4r+3; warp cw loads tile 4r + cw of
        // every chunk, one 16-byte word per lane.  Lanes poll the tiles'
        // counters in parallel (32 chunks per round) and the warp loads each
        // tile as soon as it is seen complete, so that only the last tile's
        // load is left after the source's last item finishes.  External
        // inputs are loaded the same way without polls.
        constexpr int kB = 8 / MT;  // chunks per load batch: eight loads in flight
        const int nch = (k + 511) >> 9;
        const int ntiles = k >> 7;
        const int32_t* tcnt = chained ? cp.cnt_base + P.src_cnt : nullptr;
        uint32_t mx[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          mx[m] = 0;
          keep[m][0] = make_int4(0, 0, 0, 0);
          keep[m][1] = make_int4(0, 0, 0, 0);
        }
        uint32_t xs_bits = 0;
        bool waited = true;
        for (int g0 = 0; g0 < nch && waited; g0 += 32) {
          // Chunks g0 + i (i < 32) with a tile of this warp.
          const int mine = min(32, (ntiles - cw + 3) / 4 - g0);
          uint32_t pending = mine <= 0 ? 0u : (mine >= 32 ? 0xffffffffu : (1u << mine) - 1u);
          const uint64_t t0 = global_timer_ns();
          while (pending) {
            bool ready = !chained;
            if (chained && ((pending >> lane) & 1u))
              ready = ld_acquire_gpu(tcnt + 4 * (g0 + lane) + cw) >= P.src_splits;
            uint32_t fresh_tiles = __ballot_sync(0xffffffffu, ready) & pending;
            __syncwarp();
            // The first item of the source (tile 0) published its scales.
            if (chained && cw == 0 && g0 == 0 && (fresh_tiles & 1u) && lane < MT)
              xs_bits = __float_as_uint(__ldcg(cp.xs_base + 2 * P.src + lane));
            pending &= ~fresh_tiles;
            while (fresh_tiles) {
              // Up to kB newly complete chunks per batch, loads in flight together.
              int rr[kB];
#pragma unroll
              for (int u = 0; u < kB; ++u) {
                rr[u] = fresh_tiles ? g0 + __ffs(fresh_tiles) - 1 : -1;
                fresh_tiles &= fresh_tiles - 1;
              }
              int4 vb[MT][kB];
#pragma unroll
              for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int u = 0; u < kB; ++u)
                  vb[m][u] = rr[u] >= 0
                                 ? src4[static_cast<int64_t>(m) * (k >> 2) + rr[u] * 128 + ctid]
                                 : make_int4(0, 0, 0, 0);
#pragma unroll
              for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int u = 0; u < kB; ++u) {
                  const int4 v = vb[m][u];
                  if (rr[u] == md.kc) keep[m][0] = v;
                  if (rr[u] >= 0 && rr[u] == md.kc + 1) keep[m][1] = v;
                  if (chained) {
                    mx[m] = max(mx[m], max(max(static_cast<uint32_t>(abs(v.x)), static_cast<uint32_t>(abs(v.y))),
                                           max(static_cast<uint32_t>(abs(v.z)), static_cast<uint32_t>(abs(v.w)))));
                  } else {
                    // Non-negative floats order like their bit patterns.
                    mx[m] = max(mx[m], max(max(static_cast<uint32_t>(v.x) & 0x7fffffffu,
                                               static_cast<uint32_t>(v.y) & 0x7fffffffu),
                                           max(static_cast<uint32_t>(v.z) & 0x7fffffffu,
                                               static_cast<uint32_t>(v.w) & 0x7fffffffu)));
                  }
                }
            }
            if (pending && global_timer_ns() - t0 > kWaitTimeoutNs) {
              if (lane == 0) {
                *abort_flag = 1u;
                atomicOr(&g_error_flags, kErrWaitTimeout);
              }
              waited = false;
              break;
            }
            if (pending && *abort_flag) {
              waited = false;
              break;
            }
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint32_t w = __reduce_max_sync(0xffffffffu, mx[m]);
          if (lane == 0) red[cw * 2 + m] = w;
        }
        if (cw == 0 && lane < MT) red[20 + lane] = xs_bits;
        if (!csync()) break;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (chained) xs_in[m] = __uint_as_float(red[20 + m]);
          const uint32_t mx = max(max(red[m], red[2 + m]), max(red[4 + m], red[6 + m]));
          amax[m] = chained
                        ? __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(mx)), xs_in[m]), s_src)
                        : __uint_as_float(mx);
        }
        cached_src = chained ? P.src : -1;
        cached_x = chained ? nullptr : P.x;
        cached_k = k;
      } else if (kept) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int4* row = src4 + static_cast<int64_t>(m) * (k >> 2);
          keep[m][0] = k_lo + 4 * ctid < k_hi ? row[md.kc * 128 + ctid] : make_int4(0, 0, 0, 0);
          keep[m][1] = k_lo + 512 + 4 * ctid < k_hi ? row[(md.kc + 1) * 128 + ctid]
                                                     : make_int4(0, 0, 0, 0);
        }
      }
      // Quantize the slice: q = clamp(rint(y * (127 / amax)), -127, 127),
      // and sum it for the unsigned-code correction.
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float inv = amax[m] > 0.0f ? __fdiv_rn(127.0f, amax[m]) : 0.0f;
        xsp[m] = amax[m] > 0.0f ? __fdiv_rn(amax[m], 127.0f) : 0.0f;
        const float xs_src = xs_in[m];
        const int4* row = src4 + static_cast<int64_t>(m) * (k >> 2);
        int sum = 0;
        auto quant4 = [&](int q, int4 raw) {
          float4 v;
          if (chained) {
            v.x = __fmul_rn(__fmul_rn(__int2float_rn(raw.x), xs_src), s_src);
            v.y = __fmul_rn(__fmul_rn(__int2float_rn(raw.y), xs_src), s_src);
            v.z = __fmul_rn(__fmul_rn(__int2float_rn(raw.z), xs_src), s_src);
            v.w = __fmul_rn(__fmul_rn(__int2float_rn(raw.w), xs_src), s_src);
          } else {
            v = make_float4(__int_as_float(raw.x), __int_as_float(raw.y), __int_as_float(raw.z),
                            __int_as_float(raw.w));
          }
          const int q0 = max(-127, min(127, __float2int_rn(__fmul_rn(v.x, inv))));
          const int q1 = max(-127, min(127, __float2int_rn(__fmul_rn(v.y, inv))));
          const int q2 = max(-127, min(127, __float2int_rn(__fmul_rn(v.z, inv))));
          const int q3 = max(-127, min(127, __float2int_rn(__fmul_rn(v.w, inv))));
          sum += q0 + q1 + q2 + q3;
          char4 c;
          c.x = static_cast<signed char>(q0);
          c.y = static_cast<signed char>(q1);
          c.z = static_cast<signed char>(q2);
          c.w = static_cast<signed char>(q3);
          *reinterpret_cast<char4*>(xbuf + m * xstride + q * 512 + 4 * ctid) = c;
        };
        if (kept) {
          if (k_lo + 4 * ctid < k_hi) quant4(0, keep[m][0]);
          if (k_lo + 512 + 4 * ctid < k_hi) quant4(1, keep[m][1]);
        } else {
          for (int q = 0; q < nr; ++q)
            if (k_lo + q * 512 + 4 * ctid < k_hi) quant4(q, row[(md.kc + q) * 128 + ctid]);
        }
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) red[8 + cw * 2 + m] = static_cast<uint32_t>(sum);
      }
      // The first item of a problem publishes its activation scales for the
      // problems that read its output (before it counts itself done).
      if (ctid == 0 && md.row0 == 0 && md.kc == 0)
#pragma unroll
        for (int m = 0; m < MT; ++m) cp.xs_base[2 * P.idx + m] = xsp[m];
      if (!csync()) break;
#pragma unroll
      for (int m = 0; m < MT; ++m)
        xsum[m] = static_cast<int>(red[8 + m] + red[10 + m] + red[12 + m] + red[14 + m]);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int g = 0; g < 4; ++g) a[i][m][g] = 0;
    }
    const int kblk = md.kc * 512 + 128 * cq;  // first weight of this lane's block
    if (kblk < P.k) {                          // blocks wholly past K are skipped
      uint32_t xr[MT][4][8];
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint8_t* xg = xbuf + m * xstride + (kblk - xoff) + 32 * ((j + cq) & 3);
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
        const int r = cw * 32 + rs + 8 * i;
        const uint8_t* wrow = box + r * 128;
        const uint4 w0 = *reinterpret_cast<const uint4*>(wrow + (((2 * cq) ^ rs) << 4));
        const uint4 w1 = *reinterpret_cast<const uint4*>(wrow + (((2 * cq + 1) ^ rs) << 4));
        const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
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
      // ------------------------------------------------ item end
      const int n = P.n;
      const bool whole = P.splits == 1;
      int32_t* accp = cp.acc_base + P.acc;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = md.row0 + cw * 32 + rs + 8 * i;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          int part = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) part += a[i][m][j] >> gshift[j];
          part += __shfl_xor_sync(0xffffffffu, part, 1);
          part += __shfl_xor_sync(0xffffffffu, part, 2);
          if (cq == 0 && row < n) {
            const int dot = part - xsum[m];
            const int64_t o = static_cast<int64_t>(m) * n + row;
            if (whole) {
              accp[o] = dot;
              P.y[o] = __fmul_rn(__fmul_rn(__int2float_rn(dot), xsp[m]), wscale);
              if (P.acc_out != nullptr) P.acc_out[o] = dot;
            } else {
              atomicAdd(accp + o, dot);
            }
          }
        }
      }
      // The barrier orders every thread's stores and adds before thread 0's
      // release: the counts make them visible at gpu scope (cumulatively).
      // A row tile is complete when its count reaches `splits`; with one
      // token the problem's done counter also counts the item.
      if (!csync()) break;
      if (ctid == 0) {
        int32_t* tc = cp.cnt_base + P.cnt + md.row0 / kGemvTileRows;
        if (MT == 1) red_release_gpu_add(cp.done + P.idx * kChainDoneStride, 1);
        if (!whole) *last_flag = atom_acq_rel_gpu_add(tc, 1) == P.splits - 1;
        else if (MT != 1) red_release_gpu_add(tc, 1);
      }
      if (!whole) {
        if (!csync()) break;
        if (*last_flag) {
          // The last slice of this row tile: its outputs for the caller.
          __threadfence();
          const int row = md.row0 + ctid;
          if (row < n) {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const int64_t o = static_cast<int64_t>(m) * n + row;
              const int dot = __ldcg(accp + o);
              P.y[o] = __fmul_rn(__fmul_rn(__int2float_rn(dot), xsp[m]), wscale);
              if (P.acc_out != nullptr) P.acc_out[o] = dot;
            }
          }
        }
      }
    }
  }
}

// Zeroes the chain's counters and accumulators once every earlier grid on
// the stream is done.
__global__ void __launch_bounds__(256) chain_zero_kernel(int4* p, int64_t n16) {
  grid_dependency_wait();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = make_int4(0, 0, 0, 0);
  grid_dependents_launch();
}

}  // namespace bitnet
