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
// Tile ("swap-AB"): MMA M = 128 TMEM lanes (operand A), MMA N = T tokens
// (operand B, Xq rows, K-major in shared memory), so a decode batch of 3..64
// tokens still fills the 128-row MMA.  Lanes 0..126 hold 127 weight rows as
// unsigned codes c = w + 1; lane 127 holds ones, so accumulator row 127 is
// sum_k x for every token, and acc = D[r] - D[127] is the ternary
// contraction of row r (w = c - 1).  A work item is one 127 x T output tile
// over the whole K.  Items are numbered problem by
// problem, token tile by token tile, row tile by row tile; each CTA owns one
// contiguous range of items balanced by their 512-wide K chunks, and streams
// through it without stopping between items.
//
// Roles (6 warps):
//   warp 0     TMA producer.  Two rings: packed weights, one box of 128 rows
//              x 128 bytes (a 512-wide K chunk, four I2_S blocks) per stage,
//              and activations, a T x 128-byte box of Xq per I2_S block,
//              kXB blocks per stage; both boxes use the 128-byte swizzle.
//   warp 1     TMEM allocator and MMA issuer (one thread).
//   warps 2-5  unpack and epilogue: thread r (= TMEM lane r) owns weight row
//              r of the tile.  Per block it expands its row's 32 bytes into 4
//              groups x 32 codes and stores them as 32 TMEM columns (one A
//              slot; lane 127 stores ones); a weight stage is released as soon
//              as its bytes are in registers.  At the end of an item the same
//              warps read the accumulator of their lane quarter and write
//              y = ((float)acc * xs[m]) * s, token-major; the token sums of
//              row 127 reach the other warps through shared memory.
//
// The MMA-issuing thread spends tens of cycles per small MMA, so a decode
// tile keeps the tensor pipe fed only with several issuers per SM: small
// token tiles run 3 or 4 CTAs per SM (TMEM 128 columns each).  From 33
// tokens on the library uses prefill_kernel.cuh instead (operands in shared
// memory, two accumulators); the 64- and 128-token configurations here
// remain valid.
//
// Unpack: the 32-bit word made of bytes 4i..4i+3 of a block, shifted right
// by 6-2g and masked with 0x03030303, is the four codes of weights
// 32g+4i .. 32g+4i+3 in byte order, i.e. one TMEM column of the A operand
// for the MMA over k = 32g .. 32g+31: two ALU operations per four weights,
// and no per-block work for the w = c - 1 correction, which the ones lane
// does inside the MMA.
//
// Barriers: fullw/emptyw over the weight ring (TMA -> unpack), fullx/emptyx
// over the activation ring (TMA -> MMA), afull/aempty over the TMEM A slots
// (unpack -> MMA -> unpack), dfull/dempty over the accumulator buffers
// (MMA -> epilogue -> MMA), xsum over the token sums of row 127 (warp 3 ->
// the other epilogue warps).  Every wait is bounded (ptx.cuh); there are no
// named barriers, so a timed-out wait can never leave another warp stuck.
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

constexpr int kMmaTileRows = 127;  // weight rows per tile; TMEM lane 127 holds ones

template <int T>
struct MmaCfg {
  static_assert(T == 16 || T == 32 || T == 64 || T == 128, "token tile");
  static constexpr int kRows = 128;  // MMA M
  static constexpr int kThreads = 192;
  static constexpr int kCtasPerSm = T <= 32 ? 4 : (T == 64 ? 3 : 2);
  static constexpr int kDBufs = T <= 32 ? 2 : 1;        // accumulator buffers
  static constexpr uint32_t kDCols = round32(T);        // columns of one buffer
  static constexpr int kASlots = T <= 64 ? 2 : 4;       // 32-column A slots
  static constexpr uint32_t kACol = kDBufs * kDCols;    // A slots after the buffers
  static constexpr uint32_t kTmemCols = pow2_at_least(kACol + 32u * kASlots);
  static constexpr int kWBytes = kRows * 128;           // weight box: 128 rows x 128 B
  static constexpr int kWStages = 2;
  static constexpr int kXBox = T * 128;                 // activation box: T rows x 128 B
  static constexpr int kXB = T == 16 ? 4 : (T == 32 ? 2 : 1);  // blocks per activation stage
  static constexpr int kXStageBytes = kXB * kXBox;
  static constexpr int kXStages = T <= 32 ? 2 : 4;
  static constexpr int kNumBars = 2 * kWStages + 2 * kXStages + 2 * kASlots + 2 * kDBufs + 2;
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kWStages) * kWBytes +
                                       static_cast<size_t>(kXStages) * kXStageBytes +
                                       kNumBars * 8 + 2 * T * 4 + 16;
  static constexpr uint32_t kIdesc = idesc_i8(128, T, false, true);  // u8 codes x s8
  static_assert(kTmemCols * kCtasPerSm <= 512, "tensor memory per SM");
  static_assert((kSmemBytes + 1024) * kCtasPerSm <= 228 * 1024, "shared memory per SM");
};

__device__ __forceinline__ uint32_t unpack_word(uint32_t w, int g) {
  return (w >> (6 - 2 * g)) & 0x03030303u;
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
__device__ __forceinline__ void mma_item(const BP& bp, int item, int* p, int* rt, int* tt) {
  *p = mma_find_problem(bp, item);
  const MmaProblem& P = bp.p[*p];
  const int row_tiles = (P.n + kMmaTileRows - 1) / kMmaTileRows;
  const int local = item - P.item_start;
  *tt = local / row_tiles;
  *rt = local - *tt * row_tiles;
}

template <int T, int CAP>
__global__ void __launch_bounds__(192, MmaCfg<T>::kCtasPerSm)
    i2s_mma_kernel(const __grid_constant__ MmaParamsT<CAP> bp) {
  using C = MmaCfg<T>;
  constexpr int WS = C::kWStages, XS = C::kXStages, AS = C::kASlots, DB = C::kDBufs;
  constexpr int XB = C::kXB;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* wring = smem;
  uint8_t* xring = smem + WS * C::kWBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(xring + XS * C::kXStageBytes);
  int32_t* xsum_smem = reinterpret_cast<int32_t*>(bars + C::kNumBars);  // [2][T]
  uint32_t* misc = reinterpret_cast<uint32_t*>(xsum_smem + 2 * T);     // [0] tmem, [1] abort
  volatile uint32_t* abort_flag = misc + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tokens = bp.m;

  const uint32_t bar0 = smem_u32(bars);
  auto fullw_bar = [&](int s) { return bar0 + 8u * s; };
  auto emptyw_bar = [&](int s) { return bar0 + 8u * (WS + s); };
  auto fullx_bar = [&](int s) { return bar0 + 8u * (2 * WS + s); };
  auto emptyx_bar = [&](int s) { return bar0 + 8u * (2 * WS + XS + s); };
  auto afull_bar = [&](int t) { return bar0 + 8u * (2 * WS + 2 * XS + t); };
  auto aempty_bar = [&](int t) { return bar0 + 8u * (2 * WS + 2 * XS + AS + t); };
  auto dfull_bar = [&](int b) { return bar0 + 8u * (2 * WS + 2 * XS + 2 * AS + b); };
  auto dempty_bar = [&](int b) { return bar0 + 8u * (2 * WS + 2 * XS + 2 * AS + DB + b); };
  auto xsum_bar = [&](int j) { return bar0 + 8u * (2 * WS + 2 * XS + 2 * AS + 2 * DB + j); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < WS; ++s) {
      mbar_init(fullw_bar(s), 1);
      mbar_init(emptyw_bar(s), 4);  // the four unpack warps
    }
    for (int s = 0; s < XS; ++s) {
      mbar_init(fullx_bar(s), 1);
      mbar_init(emptyx_bar(s), 1);  // MMA commit
    }
    for (int t = 0; t < AS; ++t) {
      mbar_init(afull_bar(t), 4);
      mbar_init(aempty_bar(t), 1);
    }
    for (int b = 0; b < DB; ++b) {
      mbar_init(dfull_bar(b), 1);
      mbar_init(dempty_bar(b), 4);
    }
    mbar_init(xsum_bar(0), 1);  // lane 127's thread
    mbar_init(xsum_bar(1), 1);
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
  if (warp != 0 || lane != 0) {
    if (bp.pdl) grid_dependency_wait();
    grid_dependents_launch();
  }

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      bool waited = (bp.pdl == 0);
      if (waited) grid_dependents_launch();
      int wc = 0;  // weight stages issued
      int xc = 0;  // activation stages issued
      // The weights do not depend on the preceding grid: the first WS
      // chunks' weights are requested before waiting for it, and their
      // activations right after.
      int pend_p[WS], pend_tt[WS], pend_kc[WS];
      int npend = 0;
      auto issue_x = [&](int p, int tt, int kc) -> bool {
        const MmaProblem& P = bp.p[p];
        const int nb = min(4, (P.k >> 7) - 4 * kc);
        for (int q0 = 0; q0 < nb; q0 += XB, ++xc) {
          const int s = xc % XS;
          if (xc >= XS && !mbar_wait(emptyx_bar(s), ((xc / XS) - 1) & 1, abort_flag))
            return false;
          const int nbx = min(XB, nb - q0);
          mbar_arrive_expect_tx(fullx_bar(s), nbx * C::kXBox);
          uint8_t* dst = xring + s * C::kXStageBytes;
          for (int q = 0; q < nbx; ++q)
            tma_load_2d(smem_u32(dst + q * C::kXBox), &bp.tx[p], kc * 512 + (q0 + q) * 128,
                        tt * T, fullx_bar(s));
        }
        return true;
      };
      auto wait_inputs = [&]() -> bool {
        grid_dependency_wait();
        grid_dependents_launch();
        waited = true;
        for (int i = 0; i < npend; ++i)
          if (!issue_x(pend_p[i], pend_tt[i], pend_kc[i])) return false;
        npend = 0;
        return true;
      };
      const uint64_t pol_w = l2_policy_evict_first();
      for (int item = item_lo; item < item_hi && ok; ++item) {
        int p, rt, tt;
        mma_item(bp, item, &p, &rt, &tt);
        const MmaProblem& P = bp.p[p];
        prefetch_tensormap(&bp.tw[p]);
        prefetch_tensormap(&bp.tx[p]);
        const int nk = (P.k + 511) >> 9;
        for (int kc = 0; kc < nk; ++kc, ++wc) {
          const int s = wc % WS;
          if (wc >= WS) {
            if (!waited && !wait_inputs()) {
              ok = false;
              break;
            }
            if (!mbar_wait(emptyw_bar(s), ((wc / WS) - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
          }
          mbar_arrive_expect_tx(fullw_bar(s), C::kWBytes);
          tma_load_2d_hint(smem_u32(wring + s * C::kWBytes), &bp.tw[p], kc * 128,
                           rt * kMmaTileRows, fullw_bar(s), pol_w);
          if (waited) {
            if (!issue_x(p, tt, kc)) {
              ok = false;
              break;
            }
          } else {
            pend_p[npend] = p;
            pend_tt[npend] = tt;
            pend_kc[npend] = kc;
            ++npend;
          }
        }
      }
      if (ok && !waited) ok = wait_inputs();
      // This CTA does not finish before the preceding grid has, so that the
      // completion of any grid in a chain implies that of all before it.
      grid_dependency_wait();
      if (*abort_flag || !ok) {
        *abort_flag = 1u;
        // Let the copies already issued land before shared memory goes away
        // (stages whose copies were never requested are not waited for).
        for (int i = (wc > WS ? wc - WS : 0); i < wc; ++i)
          mbar_wait(fullw_bar(i % WS), (i / WS) & 1, nullptr, kDrainTimeoutNs);
        for (int i = (xc > XS ? xc - XS : 0); i < xc; ++i)
          mbar_wait(fullx_bar(i % XS), (i / XS) & 1, nullptr, kDrainTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      int blk = 0, xc = 0, ii = 0;
      for (int item = item_lo; item < item_hi && ok; ++item, ++ii) {
        int p, rt, tt;
        mma_item(bp, item, &p, &rt, &tt);
        const MmaProblem& P = bp.p[p];
        const int b = ii % DB;
        if (ii >= DB && !mbar_wait(dempty_bar(b), ((ii / DB) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + b * C::kDCols;
        const int nk = (P.k + 511) >> 9;
        bool first = true;
        for (int kc = 0; kc < nk && ok; ++kc) {
          const int nb = min(4, (P.k >> 7) - 4 * kc);
          for (int q0 = 0; q0 < nb && ok; q0 += XB, ++xc) {
            const int s = xc % XS;
            if (!mbar_wait(fullx_bar(s), (xc / XS) & 1, abort_flag)) {
              ok = false;
              break;
            }
            const int nbx = min(XB, nb - q0);
            const uint32_t xstage = smem_u32(xring + s * C::kXStageBytes);
            for (int q = 0; q < nbx; ++q, ++blk) {
              const int t = blk % AS;
              if (!mbar_wait(afull_bar(t), (blk / AS) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              // K step g of this block: bytes 32g..32g+31 of each 128-byte Xq
              // row, i.e. the descriptor's start address plus 2g (16-byte units).
              const uint64_t bdesc = smem_desc_sw128(xstage + q * C::kXBox);
              const uint32_t acol = tmem + C::kACol + 32u * t;
              mma_i8_tmem_a(dcol, acol, bdesc, C::kIdesc, first ? 0u : 1u);
              mma_i8_tmem_a(dcol, acol + 8u, bdesc + 2u, C::kIdesc, 1u);
              mma_i8_tmem_a(dcol, acol + 16u, bdesc + 4u, C::kIdesc, 1u);
              mma_i8_tmem_a(dcol, acol + 24u, bdesc + 6u, C::kIdesc, 1u);
              first = false;
              tc_commit(aempty_bar(t));
            }
            if (ok) tc_commit(emptyx_bar(s));
          }
        }
        if (ok) tc_commit(dfull_bar(b));
      }
      // Our MMAs must be finished before TMEM is released.
      const int last = ii - 1;
      if (last >= 0)
        mbar_wait(dfull_bar(last % DB), (last / DB) & 1, nullptr,
                  ok ? kWaitTimeoutNs : kDrainTimeoutNs);
    }
  } else {
    // ------------------------------------------------- unpack and epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = true;
    int wc = 0, blk = 0, ii = 0;
    for (int item = item_lo; item < item_hi && ok; ++item, ++ii) {
      int p, rt, tt;
      mma_item(bp, item, &p, &rt, &tt);
      const MmaProblem& P = bp.p[p];
      const int nk = (P.k + 511) >> 9;
      for (int kc = 0; kc < nk && ok; ++kc, ++wc) {
        const int s = wc % WS;
        ok = __all_sync(0xffffffffu, mbar_wait(fullw_bar(s), (wc / WS) & 1, abort_flag));
        if (!ok) break;
        const int nb = min(4, (P.k >> 7) - 4 * kc);
        // Row r of the weight box: its 128 bytes (four blocks) into registers,
        // then the stage goes back to the producer.  The box was written with
        // the 128-byte swizzle: 16-byte chunk c of row r sits at c ^ (r % 8).
        const uint8_t* wrow = wring + s * C::kWBytes + r * 128;
        // Lane 127 carries ones: bytes of 0x55 unpack to code 1 in every group.
        const uint4 ones = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
        uint4 wv4[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          wv4[c] = r == kMmaTileRows ? ones
                                     : *reinterpret_cast<const uint4*>(wrow + ((c ^ (r & 7)) << 4));
        __syncwarp();
        if (lane == 0) mbar_arrive(emptyw_bar(s));
        for (int q0 = 0; q0 < nb && ok; q0 += XB) {
          const int nbx = min(XB, nb - q0);
          for (int q = 0; q < nbx; ++q, ++blk) {
            const int bi = q0 + q;  // block of the weight stage
            const uint4 c0 = wv4[2 * bi], c1 = wv4[2 * bi + 1];
            const uint32_t wv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint32_t a[32];
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
              for (int i = 0; i < 8; ++i) a[8 * g + i] = unpack_word(wv[i], g);
            const int t = blk % AS;
            if (blk >= AS) {
              // The slot's previous block has been read by its MMAs.
              ok = __all_sync(0xffffffffu,
                              mbar_wait(aempty_bar(t), ((blk / AS) - 1) & 1, abort_flag));
              if (!ok) break;
            }
            tc_fence_after();
            tmem_st_32x32b_x32(tmem + lane_base + C::kACol + 32u * t, a);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(afull_bar(t));
          }
        }
      }
      if (!ok) break;
      // ---- epilogue of this item
      const int b = ii % DB;
      ok = __all_sync(0xffffffffu, mbar_wait(dfull_bar(b), (ii / DB) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      int32_t* xsum_buf = xsum_smem + (ii & 1) * T;
      if (quarter == 3) {
        // Row 127 (this warp's lane 31) holds sum_k x of every token.
#pragma unroll 1
        for (int c0 = 0; c0 < T; c0 += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tmem + lane_base + b * C::kDCols + c0, v);
          tmem_ld_wait();
          if (lane == 31) {
#pragma unroll
            for (int j = 0; j < 16; ++j) xsum_buf[c0 + j] = static_cast<int32_t>(v[j]);
          }
        }
        if (lane == 31) mbar_arrive(xsum_bar(ii & 1));
      }
      ok = __all_sync(0xffffffffu, mbar_wait(xsum_bar(ii & 1), (ii >> 1) & 1, abort_flag));
      if (!ok) break;
      const float s = *reinterpret_cast<const float*>(P.packed + static_cast<int64_t>(P.n) * (P.k >> 2));
      const int64_t n = static_cast<int64_t>(rt) * kMmaTileRows + r;
      const int64_t tok0 = static_cast<int64_t>(tt) * T;
      const int64_t nn = P.n;
      const bool row_ok = r < kMmaTileRows && n < nn;
      float* __restrict__ yb = P.y;
      int32_t* __restrict__ ab = P.acc;
      const float* __restrict__ xsb = P.xs;
#pragma unroll 1
      for (int c0 = 0; c0 < T; c0 += 16) {
        if (tok0 + c0 >= m_tokens) break;  // warp-uniform
        float xsv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          xsv[j] = (tok0 + c0 + j < m_tokens) ? __ldg(xsb + tok0 + c0 + j) : 0.0f;
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lane_base + b * C::kDCols + c0, v);
        tmem_ld_wait();
        if (row_ok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int64_t tok = tok0 + c0 + j;
            if (tok < m_tokens) {
              const int32_t a = static_cast<int32_t>(v[j]) - xsum_buf[c0 + j];
              yb[tok * nn + n] = __fmul_rn(__fmul_rn(__int2float_rn(a), xsv[j]), s);
              if (ab != nullptr) ab[tok * nn + n] = a;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dempty_bar(b));
    }
    tmem_st_wait();  // no store of this thread outlives it
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace bitnet
