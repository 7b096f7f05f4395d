// prefill_kernel.cuh -- the I2_S ternary x int8 matmul at 33 tokens and
// more (64-token tiles up to 64 tokens, 128-token tiles up to 1024, 256-token
// tiles above) on the sm_100a tensor cores, with both MMA operands in shared
// memory and two accumulator buffers in tensor memory.
//
// Same contraction, tile and correction as the decode-sized tensor kernel
// (mma_kernel.cuh): swap-AB, MMA M = 128 rows of unsigned codes c = w + 1
// with row 127 all ones (so D[127] = sum_k x and acc = D[r] - D[127]), MMA
// N = T tokens of Xq, one 127 x T output tile over the whole K per work
// item (T = 64, 128 or 256 tokens).  What differs is where the unpacked
// weights go.  There, they are stored into tensor memory, which then has no
// room for a second accumulator, so the epilogue of a tile (tensor memory
// -> fp32 outputs) and the next tile's MMAs take turns.  Here the unpack
// warps write each 128 x 128-byte block of codes into shared memory in the
// layout the 128-byte-swizzled TMA boxes of Xq have (rows of 128 bytes,
// 16-byte chunk c of row r at c ^ (r % 8), 8-row groups 1024 bytes apart),
// and the MMA reads both operands through shared-memory descriptors ("LLM Quantization
// Paradigms: FP8, AWQ, EXL2 & BitNet b1.58 in 2026", section 5: the ternary
// contraction as a dense int8 product; "How BitNet's 1-Bit (I2_S)
// Quantization Works Compared to Standard LLM Quantization", How I2_S
// Kernels Process the Format: unpack once, reuse over many activations).
// Tensor memory then holds two T-column accumulators per CTA (at T = 256
// they take all 512 columns, so one CTA runs per SM), and a separate group
// of epilogue warps drains one while the MMAs fill the other.
//
// Roles (10 warps):
//   warp 0     TMA producer: packed weights (a 128-row x 128-byte box, four
//              I2_S blocks, per stage) and Xq (a T-token x 128-byte box
//              per block), both with the 128-byte swizzle.
//   warp 1     tensor-memory allocator and MMA issuer (one thread).
//   warps 2-5  unpack: thread r owns weight row r; per block it writes its
//              row's 128 codes as eight 16-byte chunks into an A slot, then
//              makes them visible to the tensor core (proxy fence).
//   warps 6-9  epilogue: each reads the accumulator lanes of its quarter and
//              writes y = ((float)acc * xs[m]) * s, token-major; the token
//              sums of row 127 and the tile's token scales (fetched from
//              global memory while the accumulator fills) reach the others
//              through shared memory.
//
// Barriers: fullw/emptyw (weight ring), fullx/emptyx (activation ring),
// afull/aempty (A slots: unpack -> MMA -> unpack), dfull/dempty
// (accumulators: MMA -> epilogue -> MMA), xsum (row 127's token sums and the
// tile's token scales, written to shared memory by the epilogue warps).
// Every wait is bounded (ptx.cuh).
#pragma once

#include "mma_kernel.cuh"

namespace bitnet {

// TOKENS per tile (MMA N); CTAS CTAs per SM; WSTAGES weight boxes,
// XSTAGES activation boxes and ASLOTS A slots per CTA.
template <int TOKENS, int CTAS, int WSTAGES, int XSTAGES, int ASLOTS>
struct PrefillCfgT {
  static_assert(TOKENS == 64 || TOKENS == 128 || TOKENS == 256, "token tile");
  static constexpr int T = TOKENS;            // tokens per tile (MMA N)
  static constexpr int kThreads = 320;        // 10 warps
  static constexpr int kCtasPerSm = CTAS;
  static constexpr int kDBufs = 2;            // accumulator buffers
  static constexpr uint32_t kDCols = T;       // columns of one buffer
  static constexpr uint32_t kTmemCols = pow2_at_least(2 * T);
  static constexpr int kWBytes = 128 * 128;   // weight box: 128 rows x 128 B
  static constexpr int kWStages = WSTAGES;
  static constexpr int kXBox = T * 128;       // activation box: T tokens x 128 B
  static constexpr int kXStages = XSTAGES;
  static constexpr int kABytes = 128 * 128;   // one block of codes: 128 rows x 128 B
  static constexpr int kASlots = ASLOTS;
  static constexpr int kNumBars = 2 * kWStages + 2 * kXStages + 2 * kASlots + 2 * kDBufs + 2;
  // Rings, barriers (an even count: the arrays after them stay 16-byte
  // aligned), then per accumulator buffer the token sums and token scales.
  static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kWStages) * kWBytes +
                                       static_cast<size_t>(kXStages) * kXBox +
                                       static_cast<size_t>(kASlots) * kABytes + kNumBars * 8 +
                                       2 * T * 4 + 2 * T * 4 + 16;
  static constexpr uint32_t kIdesc = idesc_i8(128, T, false, true);  // u8 codes x s8
  static_assert(kTmemCols * kCtasPerSm <= 512, "tensor memory per SM");
  static_assert((kSmemBytes + 1024) * kCtasPerSm <= 228 * 1024, "shared memory per SM");
};

// Measured on the B200 (gate 6912x2560 / down 2560x6912 at M = 2048, T =
// 128, with an earlier epilogue that fetched token scales per 16 columns):
// 2 CTAs with 1 weight stage, 3 activation stages and 2 A slots, 1.21 / 0.95
// POPS; 2 CTAs with 2 / 2 / 2, 1.20 / 0.93; 2 CTAs with 1 / 2 / 3, 1.22 /
// 0.93; 1 CTA with 2 / 6 / 4, 0.97 / 0.91.  Shared memory allows no deeper
// rings at 2 CTAs per SM.  At T = 64 the activation boxes are half the size:
// 4 stages and 3 A slots.  At T = 256 the two accumulators fill tensor
// memory, so one CTA runs per SM: 2 weight stages, 4 activation boxes of 32
// KB and 3 A slots (218 KB of shared memory); the splits 1/4/4, 2/3/5,
// 1/5/2, 1/3/6 and two 128-token boxes per stage were within 3 % of it.
template <int T>
using PrefillCfg = PrefillCfgT<T, (T == 256 ? 1 : 2), (T == 256 ? 2 : 1),
                               (T == 128 ? 3 : 4), (T == 128 ? 2 : 3)>;

// Make this thread's generic-proxy shared-memory writes visible to the
// tensor core (async proxy).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 inputs, int32 accumulators.
__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int TOK, int CAP>
__global__ void __launch_bounds__(PrefillCfg<TOK>::kThreads, PrefillCfg<TOK>::kCtasPerSm)
    i2s_prefill_kernel(const __grid_constant__ MmaParamsT<CAP> bp) {
  using C = PrefillCfg<TOK>;
  constexpr int T = C::T;
  constexpr int WS = C::kWStages, XS = C::kXStages, AS = C::kASlots, DB = C::kDBufs;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* wring = smem;
  uint8_t* xring = wring + WS * C::kWBytes;
  uint8_t* aring = xring + XS * C::kXBox;
  uint64_t* bars = reinterpret_cast<uint64_t*>(aring + AS * C::kABytes);
  int32_t* xsum_smem = reinterpret_cast<int32_t*>(bars + C::kNumBars);  // [2][T]
  float* xs_smem = reinterpret_cast<float*>(xsum_smem + 2 * T);          // [2][T]
  uint32_t* misc = reinterpret_cast<uint32_t*>(xs_smem + 2 * T);         // [0] tmem, [1] abort
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
      mbar_init(afull_bar(t), 4);   // the four unpack warps
      mbar_init(aempty_bar(t), 1);  // MMA commit
    }
    for (int b = 0; b < DB; ++b) {
      mbar_init(dfull_bar(b), 1);   // MMA commit
      mbar_init(dempty_bar(b), 4);  // the four epilogue warps
    }
    mbar_init(xsum_bar(0), 4);  // the four epilogue warps
    mbar_init(xsum_bar(1), 4);
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

  // Launch chaining as in the decode-sized kernel.
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
        for (int q = 0; q < nb; ++q, ++xc) {
          const int s = xc % XS;
          if (xc >= XS && !mbar_wait(emptyx_bar(s), ((xc / XS) - 1) & 1, abort_flag))
            return false;
          mbar_arrive_expect_tx(fullx_bar(s), C::kXBox);
          tma_load_2d(smem_u32(xring + s * C::kXBox), &bp.tx[p], kc * 512 + q * 128, tt * T,
                      fullx_bar(s));
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
      grid_dependency_wait();
      if (*abort_flag || !ok) {
        *abort_flag = 1u;
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
        const int nblk = P.k >> 7;
        for (int q = 0; q < nblk && ok; ++q, ++xc, ++blk) {
          const int s = xc % XS;
          const int t = blk % AS;
          if (!mbar_wait(fullx_bar(s), (xc / XS) & 1, abort_flag) ||
              !mbar_wait(afull_bar(t), (blk / AS) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // K step g of the block: bytes 32g..32g+31 of every 128-byte row of
          // both operands, i.e. each descriptor's start address plus 2g
          // (16-byte units).
          const uint64_t adesc = smem_desc_sw128(smem_u32(aring + t * C::kABytes));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(xring + s * C::kXBox));
#pragma unroll
          for (int g = 0; g < 4; ++g)
            mma_i8_ss(dcol, adesc + 2u * g, bdesc + 2u * g, C::kIdesc, (q == 0 && g == 0) ? 0u : 1u);
          tc_commit(aempty_bar(t));
          tc_commit(emptyx_bar(s));
        }
        if (ok) tc_commit(dfull_bar(b));
      }
      // Our MMAs must be finished before tensor memory is released.
      const int last = ii - 1;
      if (last >= 0)
        mbar_wait(dfull_bar(last % DB), (last / DB) & 1, nullptr,
                  ok ? kWaitTimeoutNs : kDrainTimeoutNs);
    }
  } else if (warp < 6) {
    // --------------------------------------------------------------- unpack
    const int r = threadIdx.x - 64;  // weight row of the tile
    uint8_t* arow = aring + (r >> 3) * 1024 + (r & 7) * 128;  // row r of an A slot
    bool ok = true;
    int wc = 0, blk = 0;
    for (int item = item_lo; item < item_hi && ok; ++item) {
      int p, rt, tt;
      mma_item(bp, item, &p, &rt, &tt);
      const MmaProblem& P = bp.p[p];
      const int nk = (P.k + 511) >> 9;
      for (int kc = 0; kc < nk && ok; ++kc, ++wc) {
        const int s = wc % WS;
        ok = __all_sync(0xffffffffu, mbar_wait(fullw_bar(s), (wc / WS) & 1, abort_flag));
        if (!ok) break;
        const int nb = min(4, (P.k >> 7) - 4 * kc);
        // Row r of the weight box (four blocks) into registers, then the
        // stage goes back to the producer.  Row 127 is the ones row: bytes
        // of 0x55 unpack to code 1 in every group.
        const uint8_t* wrow = wring + s * C::kWBytes + r * 128;
        const uint4 ones = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
        uint4 wv4[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          wv4[c] = r == kMmaTileRows ? ones
                                     : *reinterpret_cast<const uint4*>(wrow + ((c ^ (r & 7)) << 4));
        __syncwarp();
        if (lane == 0) mbar_arrive(emptyw_bar(s));
        for (int q = 0; q < nb; ++q, ++blk) {
          const int t = blk % AS;
          if (blk >= AS) {
            // The slot's previous block has been read by its MMAs.
            ok = __all_sync(0xffffffffu,
                            mbar_wait(aempty_bar(t), ((blk / AS) - 1) & 1, abort_flag));
            if (!ok) break;
          }
          const uint4 c0 = wv4[2 * q], c1 = wv4[2 * q + 1];
          const uint32_t wv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          uint8_t* dst = arow + t * C::kABytes;
          // Chunk c holds codes k = 16c .. 16c+15: group g = c / 2, words
          // 4(c % 2) .. 4(c % 2) + 3 of the block.
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int g = c >> 1, i0 = 4 * (c & 1);
            const uint4 v = make_uint4(unpack_word(wv[i0], g), unpack_word(wv[i0 + 1], g),
                                       unpack_word(wv[i0 + 2], g), unpack_word(wv[i0 + 3], g));
            *reinterpret_cast<uint4*>(dst + ((c ^ (r & 7)) << 4)) = v;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(afull_bar(t));
        }
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // tensor-memory lanes this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    constexpr int kXsPer = (T + 127) / 128;  // token scales each thread fetches
    bool ok = true;
    int ii = 0;
    for (int item = item_lo; item < item_hi && ok; ++item, ++ii) {
      int p, rt, tt;
      mma_item(bp, item, &p, &rt, &tt);
      const MmaProblem& P = bp.p[p];
      const int b = ii % DB;
      const int64_t tok0 = static_cast<int64_t>(tt) * T;
      // The tile's token scales are fetched while its accumulator fills:
      // thread r takes tokens r and r + 128.
      float xsr[kXsPer];
#pragma unroll
      for (int i = 0; i < kXsPer; ++i) {
        const int j = r + 128 * i;
        xsr[i] = (j < T && tok0 + j < m_tokens) ? __ldg(P.xs + tok0 + j) : 0.0f;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(dfull_bar(b), (ii / DB) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // Both arrays of this buffer parity were last read for item ii - 2,
      // which every epilogue warp finished before the accumulator of item
      // ii could be filled.
      int32_t* xsum_buf = xsum_smem + (ii & 1) * T;
      float* xs_buf = xs_smem + (ii & 1) * T;
#pragma unroll
      for (int i = 0; i < kXsPer; ++i) {
        const int j = r + 128 * i;
        if (j < T) xs_buf[j] = xsr[i];
      }
      if (quarter == 3) {
        // Row 127 (this warp's lane 31) holds sum_k x of every token.
#pragma unroll 1
        for (int c0 = 0; c0 < T; c0 += 32) {
          uint32_t v[16], w[16];
          tmem_ld_32x32b_x16(tmem + lane_base + b * C::kDCols + c0, v);
          tmem_ld_32x32b_x16(tmem + lane_base + b * C::kDCols + c0 + 16, w);
          tmem_ld_wait();
          if (lane == 31) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              xsum_buf[c0 + j] = static_cast<int32_t>(v[j]);
              xsum_buf[c0 + 16 + j] = static_cast<int32_t>(w[j]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(xsum_bar(ii & 1));
      ok = __all_sync(0xffffffffu, mbar_wait(xsum_bar(ii & 1), (ii >> 1) & 1, abort_flag));
      if (!ok) break;
      const float s = *reinterpret_cast<const float*>(P.packed + static_cast<int64_t>(P.n) * (P.k >> 2));
      const int64_t n = static_cast<int64_t>(rt) * kMmaTileRows + r;
      const int64_t nn = P.n;
      const bool row_ok = r < kMmaTileRows && n < nn;
      float* __restrict__ yb = P.y;
      int32_t* __restrict__ ab = P.acc;
#pragma unroll 1
      for (int c0 = 0; c0 < T; c0 += 32) {
        if (tok0 + c0 >= m_tokens) break;  // warp-uniform
        uint32_t v0[16], v1[16];
        tmem_ld_32x32b_x16(tmem + lane_base + b * C::kDCols + c0, v0);
        tmem_ld_32x32b_x16(tmem + lane_base + b * C::kDCols + c0 + 16, v1);
        tmem_ld_wait();
        if (row_ok) {
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const int4 sums = *reinterpret_cast<const int4*>(xsum_buf + c0 + 4 * g);
            const float4 scl = *reinterpret_cast<const float4*>(xs_buf + c0 + 4 * g);
            const int32_t sm[4] = {sums.x, sums.y, sums.z, sums.w};
            const float sc[4] = {scl.x, scl.y, scl.z, scl.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 4 * g + e;
              const int64_t tok = tok0 + c0 + j;
              if (tok < m_tokens) {
                const int32_t a = static_cast<int32_t>(j < 16 ? v0[j] : v1[j - 16]) - sm[e];
                yb[tok * nn + n] = __fmul_rn(__fmul_rn(__int2float_rn(a), sc[e]), s);
                if (ab != nullptr) ab[tok * nn + n] = a;
              }
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
