// bitnet_i2s.cu -- the C ABI of include/bitnet_i2s.h: argument checks on the
// host, tensor-map encoding, and the kernel launches.  One translation unit
// (the kernels are header-only) so that the device error flag is a single
// symbol.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>
#include <utility>
#include <vector>

#include "bitnet_i2s.h"
#include "bn_kernels.cuh"
#include "chain_kernel.cuh"
#include "gemv_kernel.cuh"
#include "mma_kernel.cuh"
#include "prefill_kernel.cuh"
#include "quant_kernels.cuh"

namespace {

using namespace bitnet;

constexpr int64_t kMaxK = 131072;  // 127 * K < 2^24: (float)acc is exact
constexpr int kMaxDevices = 64;

thread_local std::string g_last_error;

bitnet_status fail(bitnet_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
bitnet_status fail(bitnet_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

bitnet_status ok() {
  g_last_error.clear();
  return BITNET_OK;
}

bitnet_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BITNET_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The current device must be compute capability 10.0 (B200 class); the
// library holds sm_100a code only.
bitnet_status check_device(int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(BITNET_ERR_UNSUPPORTED, "device %d", dev);
  static std::atomic<int> verdict[kMaxDevices];  // 0 unknown, 1 ok, 2 unsupported
  int v = verdict[dev].load(std::memory_order_acquire);
  if (v == 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    v = (major == 10 && minor == 0) ? 1 : 2;
    verdict[dev].store(v, std::memory_order_release);
  }
  if (v != 1) return fail(BITNET_ERR_UNSUPPORTED, "device %d is not compute capability 10.0", dev);
  *dev_out = dev;
  return BITNET_OK;
}

// cuTensorMapEncodeTiled from the driver, without linking libcuda.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D uint8 tensor map: `cols` bytes per row (contiguous), `rows` rows with a
// pitch of `cols` bytes, box `box_cols` x `box_rows`, 128-byte swizzle.
// Out-of-bounds box elements read as zero.
bitnet_status encode_u8_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                           uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(BITNET_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BITNET_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return BITNET_OK;
}

// Raise the dynamic shared-memory limit of a kernel once per device.
template <typename Kernel>
bitnet_status ensure_smem(Kernel kern, size_t bytes, int dev, std::atomic<uint8_t>* done) {
  if (done[dev].load(std::memory_order_acquire)) return BITNET_OK;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(bytes));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  done[dev].store(1, std::memory_order_release);
  return BITNET_OK;
}

cudaLaunchAttribute pdl_attr(bool on) {
  cudaLaunchAttribute a;
  std::memset(&a, 0, sizeof(a));
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = on ? 1 : 0;
  return a;
}

bitnet_status check_matmul_args(const char* fn, const uint8_t* packed, int64_t n, int64_t k,
                                const void* x, const float* xs_or_dummy, int64_t m, float* y,
                                int64_t max_m) {
  if (packed == nullptr || x == nullptr || xs_or_dummy == nullptr || y == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "%s: null pointer argument", fn);
  if (n < 1 || m < 1) return fail(BITNET_ERR_SHAPE, "%s: N=%lld and M=%lld must be >= 1", fn,
                                  (long long)n, (long long)m);
  if (k < 128 || k % 128 != 0 || k > kMaxK)
    return fail(BITNET_ERR_SHAPE, "%s: K=%lld must be a multiple of 128 in [128, %lld]", fn,
                (long long)k, (long long)kMaxK);
  if (m > max_m)
    return fail(BITNET_ERR_SHAPE, "%s: M=%lld exceeds %lld", fn, (long long)m, (long long)max_m);
  if (n > int64_t{0x7fffffff})
    return fail(BITNET_ERR_SHAPE, "%s: N=%lld too large", fn, (long long)n);
  if (!aligned(packed, 16)) return fail(BITNET_ERR_ALIGN, "%s: packed must be 16-byte aligned", fn);
  if (!aligned(x, 16)) return fail(BITNET_ERR_ALIGN, "%s: activations must be 16-byte aligned", fn);
  if (!aligned(y, 4) || !aligned(xs_or_dummy, 4))
    return fail(BITNET_ERR_ALIGN, "%s: Y and xs must be 4-byte aligned", fn);
  return BITNET_OK;
}

int sm_count(int dev) {
  static std::atomic<int> cached[kMaxDevices];
  int v = cached[dev].load(std::memory_order_acquire);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cached[dev].store(v, std::memory_order_release);
  }
  return v;
}

// The integer-ALU kernel serves two tokens with K up to 8192 and one token
// with K up to 30720 (the activations of one problem sit in a shared-memory
// slot); everything else goes to the tensor-core kernel.
constexpr int kMaxBatch = 160;  // problems per launch: the parameter block stays under 32 KB
static_assert(sizeof(BatchParamsT<kMaxBatch>) <= 32764, "decode kernel parameter block");
// With a work queue, the share of a decode launch's stages in fixed per-CTA
// ranges; the rest is handed out at run time.
constexpr double kStaticShare = 0.7;
bool use_dp4a(int64_t m, int64_t k) {
  return (m >= 1 && m <= 2 && k <= kGemvMaxK) || (m == 1 && k <= kGemvMaxKLong);
}
// K above the short activation slot: the one-token long-K variant.
bool long_k(int64_t k) { return k > kGemvMaxK; }

// Split K of the decode kernel: at most this many (slice, row tile) items
// per launch, whose partial sums and arrival counters the workspace holds.
constexpr int64_t kSplitItemsMax = 512;

// Workspace ints of one decode launch's split area for `mt` tokens: the
// arrival counters (zeroed before the launch), then the partial sums.
size_t split_cnt_ints() { return static_cast<size_t>(kSplitItemsMax) * 4; }
size_t split_part_ints(int64_t mt) { return static_cast<size_t>(kSplitItemsMax) * 128 * mt; }

// K slices for the problems of one decode launch on `grid` CTAs.  A problem
// longer than the variant's activation slot (`max_cps` boxes of 512) is cut
// into slices that fit it.  When the launch has fewer 128-row tiles than
// CTAs, every problem's K range is cut into up to ceil(grid / tiles) slices
// of whole boxes, keeping the launch's items within kSplitItemsMax, so that
// the launch has work for every CTA.
int64_t slices_for(int64_t nk, int64_t want, int64_t max_cps) {
  int64_t sp = std::max<int64_t>((nk + max_cps - 1) / max_cps, std::min(want, nk));
  sp = std::max<int64_t>(sp, 1);
  const int64_t cps = (nk + sp - 1) / sp;
  return (nk + cps - 1) / cps;
}

template <int CAP>
void plan_splits(BatchParamsT<CAP>& bp, int64_t grid, int64_t max_cps) {
  int64_t tiles = 0;
  for (int i = 0; i < bp.count; ++i) tiles += (bp.p[i].n + kGemvTileRows - 1) / kGemvTileRows;
  int64_t want = 1;
  if (bp.split_base != nullptr && tiles < grid)
    want = std::min((grid + tiles - 1) / tiles, kSplitItemsMax / tiles);
  // Slices forced by the slot size come on top: lower `want` until the
  // launch's items fit the split area.
  for (; want > 1; --want) {
    int64_t items = 0;
    for (int i = 0; i < bp.count; ++i) {
      const int64_t nk = (bp.p[i].k + 511) / 512;
      const int64_t sp = slices_for(nk, want, max_cps);
      if (sp > 1) items += ((bp.p[i].n + kGemvTileRows - 1) / kGemvTileRows) * sp;
    }
    if (items <= kSplitItemsMax) break;
  }
  int64_t part = 0, cnt = 0;
  for (int i = 0; i < bp.count; ++i) {
    BatchProblem& q = bp.p[i];
    const int64_t nk = (q.k + 511) / 512;
    const int64_t sp = slices_for(nk, want, max_cps);
    const int64_t cps = (nk + sp - 1) / sp;
    q.splits = static_cast<int32_t>(sp);
    q.cps = static_cast<int32_t>(cps);
    q.part_off = static_cast<int32_t>(part);
    q.cnt_off = static_cast<int32_t>(cnt);
    if (sp > 1) {
      const int64_t t = (q.n + kGemvTileRows - 1) / kGemvTileRows;
      part += t * sp * bp.m * 128;
      cnt += t * 4;
    }
  }
}

// Tensor maps, work items and their stage counts for every problem.
template <int CAP>
bitnet_status plan_items(BatchParamsT<CAP>& bp, int64_t grid, int64_t max_cps) {
  if (bp.queue != nullptr) {
    // Items are handed out in order: the longest ones (largest K) first, so
    // that the last items taken are short and the CTAs end together.
    std::stable_sort(bp.p, bp.p + bp.count,
                     [](const BatchProblem& a, const BatchProblem& b) { return a.k > b.k; });
  }
  plan_splits(bp, grid, max_cps);
  int64_t items = 0, stages = 0;
  for (int i = 0; i < bp.count; ++i) {
    BatchProblem& q = bp.p[i];
    bitnet_status st = encode_u8_2d(&bp.tmap[i], q.packed, static_cast<uint64_t>(q.k / 4),
                                    static_cast<uint64_t>(q.n), 128, kGemvTileRows);
    if (st != BITNET_OK) return st;
    q.item_start = static_cast<int32_t>(items);
    q.stage_start = static_cast<int32_t>(stages);
    const int64_t tiles = (q.n + kGemvTileRows - 1) / kGemvTileRows;
    items += tiles * q.splits;
    stages += tiles * q.splits * q.cps;
    if (stages > int64_t{0x7fffffff}) return fail(BITNET_ERR_SHAPE, "too many rows in one batch");
  }
  bp.total_items = static_cast<int32_t>(items);
  bp.total_stages = static_cast<int32_t>(stages);
  // Without a queue every item sits in a fixed range; with one, the items
  // after the first kStaticShare of the stages are handed out at run time.
  bp.dyn_start = bp.total_items;
  bp.static_stages = bp.total_stages;
  if (bp.queue != nullptr) {
    const int64_t cut = static_cast<int64_t>(kStaticShare * static_cast<double>(stages));
    for (int i = 0; i < bp.count; ++i) {
      const BatchProblem& q = bp.p[i];
      const int64_t nk = q.cps;
      const int64_t tiles = ((q.n + kGemvTileRows - 1) / kGemvTileRows) * q.splits;
      if (q.stage_start + tiles * nk > cut) {
        const int64_t off = std::max<int64_t>(0, (cut - q.stage_start + nk - 1) / nk);
        bp.dyn_start = static_cast<int32_t>(q.item_start + std::min(off, tiles));
        bp.static_stages = static_cast<int32_t>(q.stage_start + std::min(off, tiles) * nk);
        break;
      }
    }
  }
  return BITNET_OK;
}

template <int MT, int CAP, int KMAX = kGemvMaxK>
bitnet_status launch_dp4a_t(BatchParamsT<CAP>& bp, cudaStream_t stream, bool pdl, int dev) {
  using C = GemvCfg<MT, KMAX>;
  static std::atomic<uint8_t> smem_done[kMaxDevices];
  auto kern = i2s_gemv_dp4a_kernel<MT, CAP, KMAX>;
  bitnet_status st = plan_items(bp, int64_t{C::kCtasPerSm} * sm_count(dev), KMAX / 512);
  if (st != BITNET_OK) return st;
  const int grid = std::min(bp.total_items, C::kCtasPerSm * sm_count(dev));
  st = ensure_smem(kern, C::kSmemBytes, dev, smem_done);
  if (st != BITNET_OK) return st;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr = pdl_attr(pdl);
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, bp);
  if (e != cudaSuccess) return cuda_fail(e, "launch of the I2_S decode kernel");
  return BITNET_OK;
}

// Persistent grid: as many CTAs as fit on the SMs, never more than row tiles.
// `pdl`: launch as a dependent of the preceding grid; `wait`: its CTAs wait
// for that grid before reading activations (skipped only when the caller
// knows the activations were complete before the preceding grid started).
// `long_variant`: problems with K > 8192 run on the long-K variant; without
// it they are cut into K slices on the standard one (which needs the split
// area of a workspace).
template <int CAP>
bitnet_status launch_dp4a(BatchParamsT<CAP>& bp, cudaStream_t stream, bool pdl, int dev,
                          bool wait = true, bool long_variant = true) {
  bp.pdl = (pdl && wait) ? 1 : 0;
  int kmax = 0;
  for (int i = 0; i < bp.count; ++i) kmax = std::max(kmax, bp.p[i].k);
  if (bp.m == 1 && long_k(kmax) && (long_variant || bp.split_base == nullptr))
    return launch_dp4a_t<1, CAP, kGemvMaxKLong>(bp, stream, pdl, dev);
  if (bp.m == 1) return launch_dp4a_t<1, CAP>(bp, stream, pdl, dev);
  return launch_dp4a_t<2, CAP>(bp, stream, pdl, dev);
}

BatchProblem make_problem(const uint8_t* packed, int64_t n, int64_t k, const int8_t* xq,
                          const float* xs, float* y, int32_t* acc) {
  BatchProblem q;
  q.packed = packed;
  q.xq = const_cast<int8_t*>(xq);
  q.xs = const_cast<float*>(xs);
  q.y = y;
  q.acc = acc;
  q.n = static_cast<int32_t>(n);
  q.k = static_cast<int32_t>(k);
  q.item_start = 0;
  q.stage_start = 0;
  q.splits = 1;
  q.cps = static_cast<int32_t>((k + 511) / 512);
  q.part_off = 0;
  q.cnt_off = 0;
  return q;
}

// ------------------------------------------------------ tensor-core path
constexpr int kMmaBatch = 96;  // problems per launch: the parameter block stays under 32 KB
static_assert(sizeof(MmaParamsT<kMmaBatch>) <= 32764, "tensor-core kernel parameter block");

// Tensor maps and item/chunk numbering for every problem of a batch.
template <int T, int CAP>
bitnet_status plan_mma(MmaParamsT<CAP>& bp, const int8_t* const* xq) {
  const int64_t token_tiles = (bp.m + T - 1) / T;
  int64_t items = 0, chunks = 0;
  for (int i = 0; i < bp.count; ++i) {
    MmaProblem& q = bp.p[i];
    bitnet_status st = encode_u8_2d(&bp.tw[i], q.packed, static_cast<uint64_t>(q.k / 4),
                                    static_cast<uint64_t>(q.n), 128, 128);
    if (st != BITNET_OK) return st;
    st = encode_u8_2d(&bp.tx[i], xq[i], static_cast<uint64_t>(q.k), static_cast<uint64_t>(bp.m),
                      128, T);
    if (st != BITNET_OK) return st;
    q.item_start = static_cast<int32_t>(items);
    q.chunk_start = static_cast<int32_t>(chunks);
    const int64_t n_items = ((q.n + kMmaTileRows - 1) / kMmaTileRows) * token_tiles;
    items += n_items;
    chunks += n_items * ((q.k + 511) / 512);
    if (chunks > int64_t{0x7fffffff}) return fail(BITNET_ERR_SHAPE, "batch too large");
  }
  bp.total_items = static_cast<int32_t>(items);
  bp.total_chunks = static_cast<int32_t>(chunks);
  return BITNET_OK;
}

template <int T, int CAP>
bitnet_status launch_mma_t(MmaParamsT<CAP>& bp, const int8_t* const* xq, cudaStream_t stream,
                           bool pdl, bool wait, int dev) {
  using C = MmaCfg<T>;
  static std::atomic<uint8_t> smem_done[kMaxDevices];
  auto kern = i2s_mma_kernel<T, CAP>;
  bitnet_status st = ensure_smem(kern, C::kSmemBytes, dev, smem_done);
  if (st != BITNET_OK) return st;
  if ((st = plan_mma<T>(bp, xq)) != BITNET_OK) return st;
  bp.pdl = (pdl && wait) ? 1 : 0;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim =
      dim3(static_cast<unsigned>(std::min(bp.total_items, C::kCtasPerSm * sm_count(dev))));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr = pdl_attr(pdl);
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, bp);
  if (e != cudaSuccess) return cuda_fail(e, "launch of the I2_S tensor-core kernel");
  return BITNET_OK;
}

// The prefill kernel: tiles of T tokens, both operands in shared memory.
template <int T, int CAP>
bitnet_status launch_prefill(MmaParamsT<CAP>& bp, const int8_t* const* xq, cudaStream_t stream,
                             bool pdl, bool wait, int dev) {
  using C = PrefillCfg<T>;
  static std::atomic<uint8_t> smem_done[kMaxDevices];
  auto kern = i2s_prefill_kernel<T, CAP>;
  bitnet_status st = ensure_smem(kern, C::kSmemBytes, dev, smem_done);
  if (st != BITNET_OK) return st;
  if ((st = plan_mma<C::T>(bp, xq)) != BITNET_OK) return st;
  bp.pdl = (pdl && wait) ? 1 : 0;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim =
      dim3(static_cast<unsigned>(std::min(bp.total_items, C::kCtasPerSm * sm_count(dev))));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr = pdl_attr(pdl);
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, bp);
  if (e != cudaSuccess) return cuda_fail(e, "launch of the I2_S prefill kernel");
  return BITNET_OK;
}

// Token tile by M, as measured best: 16 or 32 tokens on the TMEM-A kernel
// (4 CTAs per SM); 64 tokens on the shared-memory kernel (large layer at
// M = 64: 1.52 TB/s against 1.25 on the TMEM-A kernel at 64 tokens); 128
// tokens up to M = 1024 (64-token tiles there lose more to unpacking per MAC
// than they gain in tiles: gate 6912x2560 at M = 512, 0.56 against 0.68
// POPS); 256 tokens above, one CTA per SM (gate + up + down 6912x2560 /
// 2560x6912 at M = 2048: 160 against 166 us per set; at M = 1024 the two
// tie, at M = 512 the 128-token tile is 8 % faster).
template <int CAP>
bitnet_status launch_mma(MmaParamsT<CAP>& bp, const int8_t* const* xq, cudaStream_t stream,
                         bool pdl, bool wait, int dev) {
  if (bp.m <= 16) return launch_mma_t<16>(bp, xq, stream, pdl, wait, dev);
  if (bp.m <= 32) return launch_mma_t<32>(bp, xq, stream, pdl, wait, dev);
  if (bp.m <= 64) return launch_prefill<64>(bp, xq, stream, pdl, wait, dev);
  if (bp.m <= 1024) return launch_prefill<128>(bp, xq, stream, pdl, wait, dev);
  return launch_prefill<256>(bp, xq, stream, pdl, wait, dev);
}

MmaProblem make_mma_problem(const uint8_t* packed, int64_t n, int64_t k, const float* xs, float* y,
                            int32_t* acc) {
  MmaProblem q;
  q.packed = packed;
  q.xs = xs;
  q.y = y;
  q.acc = acc;
  q.n = static_cast<int32_t>(n);
  q.k = static_cast<int32_t>(k);
  q.item_start = 0;
  q.chunk_start = 0;
  return q;
}

// One problem, on whichever kernel serves its shape.
bitnet_status run_matmul(const uint8_t* packed, int64_t n, int64_t k, const int8_t* xq,
                         const float* xs, int64_t m, float* y, int32_t* acc, bool pdl,
                         cudaStream_t stream, int dev) {
  if (use_dp4a(m, k)) {
    BatchParamsT<1> bp;
    bp.count = 1;
    bp.m = static_cast<int32_t>(m);
    bp.queue = nullptr;
    bp.split_base = nullptr;
    bp.cnt_base = nullptr;
    bp.p[0] = make_problem(packed, n, k, xq, xs, y, acc);
    return launch_dp4a(bp, stream, pdl, dev);
  }
  MmaParamsT<1> bp;
  bp.count = 1;
  bp.m = static_cast<int32_t>(m);
  bp.p[0] = make_mma_problem(packed, n, k, xs, y, acc);
  const int8_t* xqs[1] = {xq};
  return launch_mma(bp, xqs, stream, pdl, true, dev);
}

// Many tensor-core problems sharing M: launches of at most kMmaBatch
// problems in chunks of equal size, the first waiting for the preceding grid
// (when `pdl`), the later ones dependent launches that skip the wait, as for
// the decode batches.
bitnet_status run_mma_batches(const std::vector<MmaProblem>& probs,
                              const std::vector<const int8_t*>& xqs, int64_t m, bool pdl,
                              cudaStream_t stream, int dev, bool wait_first = true) {
  static thread_local MmaParamsT<kMmaBatch> bp;
  const size_t total = probs.size();
  if (total == 0) return BITNET_OK;
  const size_t nchunks = (total + kMmaBatch - 1) / kMmaBatch;
  for (size_t c = 0; c < nchunks; ++c) {
    const size_t lo = total * c / nchunks;
    const size_t hi = total * (c + 1) / nchunks;
    bp.count = static_cast<int32_t>(hi - lo);
    bp.m = static_cast<int32_t>(m);
    for (size_t i = lo; i < hi; ++i) bp.p[i - lo] = probs[i];
    bitnet_status st = launch_mma(bp, xqs.data() + lo, stream, c == 0 ? pdl : true,
                                  c == 0 && wait_first, dev);
    if (st != BITNET_OK) return st;
  }
  return BITNET_OK;
}

constexpr int64_t kMaxTokens = int64_t{65535} * 16;  // grid.y limit at the smallest tile

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// Workspace of one problem's quantized activations: M x K int8, then M
// fp32 scales.
size_t slot_bytes(int64_t m, int64_t k) {
  return align256(static_cast<size_t>(m) * static_cast<size_t>(k)) +
         align256(static_cast<size_t>(m) * sizeof(float));
}

// Decode launches of a batch of `count` problems at most (the two kernel
// variants are chunked separately, hence one launch more when there are two
// problems or more).
size_t decode_launches(int count) {
  return static_cast<size_t>((count + kMaxBatch - 1) / kMaxBatch + (count > 1 ? 1 : 0));
}

// The workspace after the activation slots: per decode launch a work
// counter; for up to two tokens also per launch the split arrival counters
// (all of them zeroed before the launches), then the split partial sums.
size_t decode_tail_bytes(int count, int64_t m) {
  const size_t nl = decode_launches(count);
  const bool split = m <= 2;
  size_t b = align256(sizeof(int32_t) * (nl + (split ? nl * split_cnt_ints() : 0)));
  if (split) b += align256(sizeof(int32_t) * nl * split_part_ints(m));
  return b;
}

struct DecodeTail {
  int32_t* zero = nullptr;   // counters to zero before the decode launches
  size_t zero_ints = 0;
  int32_t* queue = nullptr;  // per launch: work counter
  int32_t* cnt = nullptr;    // per launch: split_cnt_ints() arrival counters
  int32_t* part = nullptr;   // per launch: split_part_ints(m) partial sums
  int64_t m = 0;

  template <int CAP>
  void assign(BatchParamsT<CAP>& bp, size_t launch) const {
    bp.queue = queue != nullptr ? queue + launch : nullptr;
    bp.cnt_base = cnt != nullptr ? cnt + launch * split_cnt_ints() : nullptr;
    bp.split_base = part != nullptr ? part + launch * split_part_ints(m) : nullptr;
  }
};

// The decode tail at `base` (null: no workspace) for `count` problems of at
// most `m` tokens.
DecodeTail decode_tail(void* base, int count, int64_t m) {
  DecodeTail t;
  if (base == nullptr) return t;
  const size_t nl = decode_launches(count);
  const bool split = m <= 2;
  int32_t* w = static_cast<int32_t*>(base);
  t.zero = w;
  t.zero_ints = nl + (split ? nl * split_cnt_ints() : 0);
  t.queue = w;
  if (split) {
    t.cnt = w + nl;
    t.part = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(base) +
                                        align256(sizeof(int32_t) * t.zero_ints));
    t.m = m;
  }
  return t;
}

// One decode launch: problems [lo, hi) of the index list, and its variant.
struct DecodeChunk {
  size_t lo, hi;
  bool long_variant;  // K > 8192 on the long-K variant (else sliced)
};

// Cuts the decode problems (indices into a batch; `nk_of(i)` gives problem
// i's N and K) into launches of at most kMaxBatch problems, in chunks of
// equal size.  With a split area (`can_slice`), one-token problems with
// K > 8192 run in K slices on the standard variant, as many as the split
// area holds.  The others run on the long-K variant: when they have fewer
// 128-row tiles than that variant keeps CTAs on the GPU, every problem
// joins them there, so the launch still has work for every CTA; otherwise
// the two kinds get separate launches.
template <typename NKOf>
std::vector<DecodeChunk> decode_chunks(std::vector<int>& idx, NKOf nk_of, int dev,
                                       bool can_slice) {
  int64_t sliced_items = 0;
  auto short_or_sliced = [&](int i) {
    const auto nk = nk_of(i);
    if (!long_k(nk.second)) return true;
    if (!can_slice) return false;
    const int64_t items = ((nk.first + kGemvTileRows - 1) / kGemvTileRows) *
                          slices_for((nk.second + 511) / 512, 1, kGemvMaxK / 512);
    if (sliced_items + items > kSplitItemsMax) return false;
    sliced_items += items;
    return true;
  };
  const auto mid = std::stable_partition(idx.begin(), idx.end(), short_or_sliced);
  size_t split = static_cast<size_t>(mid - idx.begin());
  int64_t long_tiles = 0;
  for (size_t j = split; j < idx.size(); ++j)
    long_tiles += (nk_of(idx[j]).first + kGemvTileRows - 1) / kGemvTileRows;
  const int64_t long_ctas =
      static_cast<int64_t>(GemvCfg<1, kGemvMaxKLong>::kCtasPerSm) * sm_count(dev);
  if (split < idx.size() && long_tiles < long_ctas) split = 0;  // one group
  std::vector<DecodeChunk> out;
  for (const auto& g : {std::make_pair(size_t{0}, split), std::make_pair(split, idx.size())}) {
    const size_t n = g.second - g.first;
    if (n == 0) continue;
    const bool long_variant = g.first == split || split == 0;
    const size_t nchunks = (n + kMaxBatch - 1) / kMaxBatch;
    for (size_t c = 0; c < nchunks; ++c)
      out.push_back({g.first + n * c / nchunks, g.first + n * (c + 1) / nchunks, long_variant});
  }
  return out;
}

// Quantizer launch(es) and matmul launches of a batch of fused problems on a
// workspace laid out as bitnet_i2s_quant_gemv_batched_workspace_bytes says:
// the problems' activation slots, then the decode tail.
//  1. One launch quantizes every problem's tokens into the workspace (and
//     zeroes the decode launches' counters).
//  2. Problems the integer-ALU decode kernel serves (M <= 2, K <= 8192, or
//     M = 1 with K <= 30720) run in launches of at most kMaxBatch problems,
//     the rest in launches of at most kMmaBatch problems on the tensor-core
//     kernel.
// The first matmul launch waits for the quantizer; every later one is a
// dependent launch that skips the wait and starts streaming as soon as SMs
// free up: each launch in the chain starts only after every thread of the
// one before it has signalled, which the first launch's threads do only
// after their wait, so all of them start after the quantizer has finished;
// no matmul writes what another reads; and every CTA waits for the grid
// before its own before it exits, so the last launch completes last.
bitnet_status run_quant_batched(const bitnet_i2s_problem* problems, int count, int64_t M,
                                void* workspace, cudaStream_t s, int dev) {
  static thread_local QuantBatchParams qp;         // 32 KB: kept off the stack
  static thread_local BatchParamsT<kMaxBatch> bp;  // 32 KB
  std::vector<std::pair<int8_t*, float*>> sl(static_cast<size_t>(count));
  uint8_t* w = static_cast<uint8_t*>(workspace);
  for (int i = 0; i < count; ++i) {
    sl[i] = {reinterpret_cast<int8_t*>(w),
             reinterpret_cast<float*>(w + align256(static_cast<size_t>(M) * problems[i].K))};
    w += slot_bytes(M, problems[i].K);
  }
  const DecodeTail tail = decode_tail(w, count, M);
  for (int base = 0; base < count; base += kQuantBatch) {
    const int cnt = std::min(kQuantBatch, count - base);
    qp.count = cnt;
    qp.m = static_cast<int32_t>(M);
    // The first quantizer launch zeroes the counters; every decode launch
    // reads them only once the quantizers have finished.
    qp.queue = base == 0 ? tail.zero : nullptr;
    qp.nqueue = base == 0 ? static_cast<int32_t>(tail.zero_ints) : 0;
    for (int i = 0; i < cnt; ++i) {
      qp.p[i].x = problems[base + i].X;
      qp.p[i].xq = sl[base + i].first;
      qp.p[i].xs = sl[base + i].second;
      qp.p[i].k = problems[base + i].K;
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(cnt * M));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr = pdl_attr(true);
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, act_quant_batched_kernel, qp);
    if (e != cudaSuccess) return cuda_fail(e, "launch of the batched activation quant kernel");
  }
  std::vector<int> small;
  std::vector<MmaProblem> big;
  std::vector<const int8_t*> big_xq;
  for (int i = 0; i < count; ++i) {
    const bitnet_i2s_problem& q = problems[i];
    if (use_dp4a(M, q.K)) {
      small.push_back(i);
    } else {
      big.push_back(make_mma_problem(q.packed, q.N, q.K, sl[i].second, q.Y, q.acc_or_null));
      big_xq.push_back(sl[i].first);
    }
  }
  bool first = true;
  if (!small.empty()) {
    const auto chunks = decode_chunks(
        small, [&](int i) { return std::make_pair(problems[i].N, problems[i].K); }, dev,
        tail.part != nullptr);
    for (size_t c = 0; c < chunks.size(); ++c) {
      const size_t lo = chunks[c].lo;
      const size_t hi = chunks[c].hi;
      bp.count = static_cast<int32_t>(hi - lo);
      bp.m = static_cast<int32_t>(M);
      tail.assign(bp, c);
      for (size_t i = lo; i < hi; ++i) {
        const bitnet_i2s_problem& q = problems[small[i]];
        bp.p[i - lo] = make_problem(q.packed, q.N, q.K, sl[small[i]].first, sl[small[i]].second,
                                    q.Y, q.acc_or_null);
      }
      bitnet_status st = launch_dp4a(bp, s, /*pdl=*/true, dev, /*wait=*/first,
                                     chunks[c].long_variant);
      if (st != BITNET_OK) return st;
      first = false;
    }
  }
  if (!big.empty()) {
    // run_mma_batches waits in its first launch only when asked to.
    bitnet_status st = run_mma_batches(big, big_xq, M, /*pdl=*/true, s, dev, /*wait_first=*/first);
    if (st != BITNET_OK) return st;
  }
  return BITNET_OK;
}

}  // namespace

extern "C" {

size_t bitnet_i2s_packed_bytes(int64_t N, int64_t K) {
  if (N < 1 || K < 128 || K % 128 != 0) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K) / 4 + 4;
}

bitnet_status bitnet_i2s_pack(const float* W, int64_t N, int64_t K, uint8_t* packed,
                              void* stream) {
  if (W == nullptr || packed == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_pack: null pointer argument");
  if (N < 1 || K < 128 || K % 128 != 0 || K > kMaxK)
    return fail(BITNET_ERR_SHAPE, "bitnet_i2s_pack: N=%lld, K=%lld (K a multiple of 128)",
                (long long)N, (long long)K);
  if (!aligned(W, 16) || !aligned(packed, 16))
    return fail(BITNET_ERR_ALIGN, "bitnet_i2s_pack: W and packed must be 16-byte aligned");
  int dev;
  bitnet_status st = check_device(&dev);
  if (st != BITNET_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t count = N * K;
  uint8_t* tail = packed + count / 4;
  cudaError_t e = cudaMemsetAsync(tail, 0, 4, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t n4 = count / 4;
  const int grid_a = static_cast<int>(std::min<int64_t>((n4 + 255) / 256, int64_t{sms} * 8));
  i2s_absmax_kernel<<<grid_a, 256, 0, s>>>(reinterpret_cast<const float4*>(W), n4,
                                           reinterpret_cast<unsigned int*>(tail));
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the absmax kernel");
  const int64_t words = count / 16;
  const int grid_p = static_cast<int>(std::min<int64_t>((words + 255) / 256, int64_t{sms} * 16));
  i2s_pack_kernel<<<grid_p, 256, 0, s>>>(W, words, reinterpret_cast<uint32_t*>(packed),
                                         reinterpret_cast<const float*>(tail));
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the pack kernel");
  return ok();
}

bitnet_status bitnet_act_quant_i8(const float* X, int64_t M, int64_t K, int8_t* Xq, float* xs,
                                  void* stream) {
  if (X == nullptr || Xq == nullptr || xs == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_act_quant_i8: null pointer argument");
  if (M < 1 || M > int64_t{0x7fffffff} || K < 16 || K % 16 != 0 || K > kMaxK)
    return fail(BITNET_ERR_SHAPE, "bitnet_act_quant_i8: M=%lld, K=%lld (K a multiple of 16)",
                (long long)M, (long long)K);
  if (!aligned(X, 16) || !aligned(Xq, 16) || !aligned(xs, 4))
    return fail(BITNET_ERR_ALIGN, "bitnet_act_quant_i8: X and Xq must be 16-byte aligned");
  int dev;
  bitnet_status st = check_device(&dev);
  if (st != BITNET_OK) return st;
  act_quant_kernel<<<static_cast<unsigned>(M), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      X, K, Xq, xs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the activation quant kernel");
  return ok();
}

bitnet_status bitnet_i2s_gemv(const uint8_t* packed, int64_t N, int64_t K, const int8_t* Xq,
                              const float* xs, int64_t M, float* Y, int32_t* acc_or_null,
                              void* stream) {
  bitnet_status st = check_matmul_args("bitnet_i2s_gemv", packed, N, K, Xq, xs, M, Y, 64);
  if (st != BITNET_OK) return st;
  int dev;
  if ((st = check_device(&dev)) != BITNET_OK) return st;
  st = run_matmul(packed, N, K, Xq, xs, M, Y, acc_or_null, false,
                  static_cast<cudaStream_t>(stream), dev);
  return st == BITNET_OK ? ok() : st;
}

bitnet_status bitnet_i2s_gemm(const uint8_t* packed, int64_t N, int64_t K, const int8_t* Xq,
                              const float* xs, int64_t M, float* Y, int32_t* acc_or_null,
                              void* stream) {
  bitnet_status st = check_matmul_args("bitnet_i2s_gemm", packed, N, K, Xq, xs, M, Y, kMaxTokens);
  if (st != BITNET_OK) return st;
  int dev;
  if ((st = check_device(&dev)) != BITNET_OK) return st;
  st = run_matmul(packed, N, K, Xq, xs, M, Y, acc_or_null, false,
                  static_cast<cudaStream_t>(stream), dev);
  return st == BITNET_OK ? ok() : st;
}

bitnet_status bitnet_i2s_dequant_f32(const uint8_t* packed, int64_t N, int64_t K, float* W_out,
                                     void* stream) {
  if (packed == nullptr || W_out == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_dequant_f32: null pointer argument");
  if (N < 1 || K < 128 || K % 128 != 0 || K > kMaxK)
    return fail(BITNET_ERR_SHAPE, "bitnet_i2s_dequant_f32: N=%lld, K=%lld (K a multiple of 128)",
                (long long)N, (long long)K);
  if (!aligned(packed, 16) || !aligned(W_out, 16))
    return fail(BITNET_ERR_ALIGN, "bitnet_i2s_dequant_f32: packed and W_out must be 16-byte aligned");
  int dev;
  bitnet_status st = check_device(&dev);
  if (st != BITNET_OK) return st;
  const int64_t words = N * K / 16;
  const int grid = static_cast<int>(std::min<int64_t>((words + 255) / 256, int64_t{sm_count(dev)} * 16));
  i2s_dequant_f32_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(packed), words,
      reinterpret_cast<const float*>(packed + N * K / 4), W_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the dequantize kernel");
  return ok();
}

size_t bitnet_ternarize_absmean_workspace_bytes(void) {
  return static_cast<size_t>(kAbsMeanBlocks) * sizeof(double);
}

bitnet_status bitnet_ternarize_absmean(const float* W, int64_t count, double eps, float* W_out,
                                       double* gamma_out, void* workspace, size_t workspace_bytes,
                                       void* stream) {
  if (W == nullptr || W_out == nullptr || gamma_out == nullptr || workspace == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_ternarize_absmean: null pointer argument");
  if (count < 1) return fail(BITNET_ERR_SHAPE, "bitnet_ternarize_absmean: count=%lld", (long long)count);
  if (!(eps >= 0.0)) return fail(BITNET_ERR_INVALID_ARG, "bitnet_ternarize_absmean: eps must be >= 0");
  if (workspace_bytes < bitnet_ternarize_absmean_workspace_bytes())
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_ternarize_absmean: workspace of %zu bytes < %zu",
                workspace_bytes, bitnet_ternarize_absmean_workspace_bytes());
  if (!aligned(W, 4) || !aligned(W_out, 4) || !aligned(gamma_out, 8) || !aligned(workspace, 8))
    return fail(BITNET_ERR_ALIGN, "bitnet_ternarize_absmean: misaligned pointer");
  int dev;
  bitnet_status st = check_device(&dev);
  if (st != BITNET_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* partial = static_cast<double*>(workspace);
  absmean_partial_kernel<<<kAbsMeanBlocks, 256, 0, s>>>(W, count, partial);
  absmean_finish_kernel<<<1, 32, 0, s>>>(partial, kAbsMeanBlocks, count, gamma_out);
  const int grid = static_cast<int>(std::min<int64_t>((count + 255) / 256, int64_t{sm_count(dev)} * 16));
  ternarize_kernel<<<grid, 256, 0, s>>>(W, count, eps, gamma_out, W_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the ternarization kernels");
  return ok();
}

size_t bitnet_i2s_quant_gemv_workspace_bytes(int64_t M, int64_t K) {
  if (M < 1 || K < 128 || K % 128 != 0) return 0;
  return slot_bytes(M, K) + decode_tail_bytes(1, M);
}

bitnet_status bitnet_i2s_quant_gemv(const uint8_t* packed, int64_t N, int64_t K, const float* X,
                                    int64_t M, float* Y, int32_t* acc_or_null, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  const float* dummy_xs = reinterpret_cast<const float*>(X);
  bitnet_status st =
      check_matmul_args("bitnet_i2s_quant_gemv", packed, N, K, X, dummy_xs, M, Y, kMaxTokens);
  if (st != BITNET_OK) return st;
  if (workspace == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_quant_gemv: null workspace");
  if (!aligned(workspace, 256))
    return fail(BITNET_ERR_ALIGN, "bitnet_i2s_quant_gemv: workspace must be 256-byte aligned");
  const size_t need = bitnet_i2s_quant_gemv_workspace_bytes(M, K);
  if (workspace_bytes < need)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_quant_gemv: workspace of %zu bytes < %zu",
                workspace_bytes, need);
  int dev;
  if ((st = check_device(&dev)) != BITNET_OK) return st;
  // One problem of the batched path: its workspace layout is the batched
  // layout for one problem.
  bitnet_i2s_problem q;
  q.packed = packed;
  q.N = N;
  q.K = K;
  q.X = X;
  q.Y = Y;
  q.acc_or_null = acc_or_null;
  st = run_quant_batched(&q, 1, M, workspace, static_cast<cudaStream_t>(stream), dev);
  return st == BITNET_OK ? ok() : st;
}

size_t bitnet_i2s_quant_gemv_batched_workspace_bytes(const bitnet_i2s_problem* problems,
                                                     int count, int64_t M) {
  if (problems == nullptr || count < 1 || M < 1) return 0;
  size_t total = 0;
  for (int i = 0; i < count; ++i) {
    const int64_t k = problems[i].K;
    if (k < 128 || k % 128 != 0) return 0;
    total += slot_bytes(M, k);
  }
  return total + decode_tail_bytes(count, M);
}

bitnet_status bitnet_i2s_quant_gemv_batched(const bitnet_i2s_problem* problems, int count,
                                            int64_t M, void* workspace, size_t workspace_bytes,
                                            void* stream) {
  if (problems == nullptr || count < 1)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_quant_gemv_batched: no problems");
  if (M < 1 || M > kMaxTokens)
    return fail(BITNET_ERR_SHAPE, "bitnet_i2s_quant_gemv_batched: M=%lld", (long long)M);
  for (int i = 0; i < count; ++i) {
    const bitnet_i2s_problem& q = problems[i];
    bitnet_status st = check_matmul_args("bitnet_i2s_quant_gemv_batched", q.packed, q.N, q.K, q.X,
                                         q.X, M, q.Y, kMaxTokens);
    if (st != BITNET_OK) return st;
  }
  if (workspace == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_quant_gemv_batched: null workspace");
  if (!aligned(workspace, 256))
    return fail(BITNET_ERR_ALIGN,
                "bitnet_i2s_quant_gemv_batched: workspace must be 256-byte aligned");
  const size_t need = bitnet_i2s_quant_gemv_batched_workspace_bytes(problems, count, M);
  if (workspace_bytes < need)
    return fail(BITNET_ERR_INVALID_ARG,
                "bitnet_i2s_quant_gemv_batched: workspace of %zu bytes < %zu", workspace_bytes,
                need);
  int dev;
  bitnet_status st = check_device(&dev);
  if (st != BITNET_OK) return st;
  st = run_quant_batched(problems, count, M, workspace, static_cast<cudaStream_t>(stream), dev);
  return st == BITNET_OK ? ok() : st;
}

size_t bitnet_i2s_gemv_batched_workspace_bytes(int count) {
  // The token count is not known here: the split area is sized for the
  // decode kernel's largest, two tokens.
  return count < 1 ? 0 : decode_tail_bytes(count, 2);
}

bitnet_status bitnet_i2s_gemv_batched(const bitnet_i2s_qproblem* problems, int count, int64_t M,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  if (problems == nullptr || count < 1)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_gemv_batched: no problems");
  if (M < 1 || M > kMaxTokens)
    return fail(BITNET_ERR_SHAPE, "bitnet_i2s_gemv_batched: M=%lld", (long long)M);
  for (int i = 0; i < count; ++i) {
    const bitnet_i2s_qproblem& q = problems[i];
    bitnet_status st = check_matmul_args("bitnet_i2s_gemv_batched", q.packed, q.N, q.K, q.Xq,
                                         q.xs, M, q.Y, kMaxTokens);
    if (st != BITNET_OK) return st;
  }
  if (workspace != nullptr) {
    if (!aligned(workspace, 256))
      return fail(BITNET_ERR_ALIGN, "bitnet_i2s_gemv_batched: workspace must be 256-byte aligned");
    if (workspace_bytes < bitnet_i2s_gemv_batched_workspace_bytes(count))
      return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_gemv_batched: workspace of %zu bytes < %zu",
                  workspace_bytes, bitnet_i2s_gemv_batched_workspace_bytes(count));
  }
  int dev;
  bitnet_status st = check_device(&dev);
  if (st != BITNET_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Decode-kernel problems in launches of at most kMaxBatch, tensor-core
  // problems in launches of at most kMmaBatch.  The first launch is
  // ordinary, or, with a workspace, the grid that zeroes its counters after
  // waiting for all earlier work on the stream; either way nothing later
  // starts before that work has finished.  The later launches are dependent
  // launches that start as SMs free up.
  static thread_local BatchParamsT<kMaxBatch> bp;
  std::vector<int> small;
  std::vector<MmaProblem> big;
  std::vector<const int8_t*> big_xq;
  for (int i = 0; i < count; ++i) {
    const bitnet_i2s_qproblem& q = problems[i];
    if (use_dp4a(M, q.K)) {
      small.push_back(i);
    } else {
      big.push_back(make_mma_problem(q.packed, q.N, q.K, q.xs, q.Y, q.acc_or_null));
      big_xq.push_back(q.Xq);
    }
  }
  const DecodeTail tail = decode_tail(workspace, count, 2);
  bool first = true;
  if (!small.empty()) {
    const auto chunks = decode_chunks(
        small, [&](int i) { return std::make_pair(problems[i].N, problems[i].K); }, dev,
        tail.part != nullptr);
    const size_t nchunks = chunks.size();
    if (workspace != nullptr) {
      // One grid zeroes the counters once the work before this call is done;
      // the first decode launch reads them after waiting for it.
      cudaLaunchConfig_t cfg;
      std::memset(&cfg, 0, sizeof(cfg));
      cfg.gridDim = dim3(1);
      cfg.blockDim = dim3(256);
      cfg.stream = s;
      cudaLaunchAttribute attr = pdl_attr(true);
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      cudaError_t e = cudaLaunchKernelEx(&cfg, zero_counters_kernel, tail.zero,
                                         static_cast<int32_t>(tail.zero_ints));
      if (e != cudaSuccess) return cuda_fail(e, "launch of the counter reset");
    }
    for (size_t c = 0; c < nchunks; ++c) {
      const size_t lo = chunks[c].lo;
      const size_t hi = chunks[c].hi;
      bp.count = static_cast<int32_t>(hi - lo);
      bp.m = static_cast<int32_t>(M);
      tail.assign(bp, c);
      for (size_t i = lo; i < hi; ++i) {
        const bitnet_i2s_qproblem& q = problems[small[i]];
        bp.p[i - lo] = make_problem(q.packed, q.N, q.K, q.Xq, q.xs, q.Y, q.acc_or_null);
      }
      const bool after_reset = workspace != nullptr && c == 0;
      st = launch_dp4a(bp, s, /*pdl=*/!first || after_reset, dev, /*wait=*/after_reset,
                       chunks[c].long_variant);
      if (st != BITNET_OK) return st;
      first = false;
    }
  }
  if (!big.empty()) {
    st = run_mma_batches(big, big_xq, M, /*pdl=*/!first, s, dev, /*wait_first=*/false);
    if (st != BITNET_OK) return st;
  }
  return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of bitnet_i2s_quant_gemv.  Some callers have no way
// to hand the library device scratch: a C plug-in that only receives raw
// input and output pointers from a host framework that owns every allocation,
// or a latency-critical loop that must never call the CUDA allocator (a
// cudaMalloc can synchronize the device).  For them the scratch lives in a
// fixed array in this library's device image, so every GPU that loads the
// library holds it (1 MiB) until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t{1} << 20;

}  // namespace

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// cuCtxGetCurrent from the driver, without linking libcuda.
PFN_cuCtxGetCurrent_v4000 ctx_fn() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  return fn;
}

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address must come
// from the runtime.  It is looked up once per device and context, with the
// device current: a device reset destroys the context that held the library's
// device image, and the next call sees a new context and looks the address up
// again instead of using the old one.
bitnet_status noalloc_scratch(int dev, void** out) {
  struct Entry {
    CUcontext ctx;
    void* ptr;
  };
  static std::mutex mu;
  static Entry cached[kMaxDevices];
  CUcontext ctx = nullptr;
  // The runtime call below makes the device's primary context current if no
  // context is yet, so the context is read after it on a first call.
  auto get_ctx = ctx_fn();
  std::lock_guard<std::mutex> lock(mu);
  if (get_ctx != nullptr && get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  if (cached[dev].ptr == nullptr || ctx == nullptr || cached[dev].ctx != ctx) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
    if (p == nullptr) return fail(BITNET_ERR_CUDA, "static scratch has no device address");
    if (get_ctx != nullptr && get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    cached[dev].ptr = p;
    cached[dev].ctx = ctx;  // null: unknown, looked up again on the next call
  }
  *out = cached[dev].ptr;
  return BITNET_OK;
}

}  // namespace

extern "C" {

bitnet_status bitnet_i2s_quant_gemv_noalloc(const uint8_t* packed, int64_t N, int64_t K,
                                            const float* X, int64_t M, float* Y,
                                            int32_t* acc_or_null, void* stream) {
  const size_t need = bitnet_i2s_quant_gemv_workspace_bytes(M, K);
  if (need != 0 && need > kNoAllocScratchBytes)
    return fail(BITNET_ERR_SHAPE,
                "bitnet_i2s_quant_gemv_noalloc: M=%lld x K=%lld needs %zu scratch bytes, more "
                "than the %zu-byte static scratch (use bitnet_i2s_quant_gemv with a workspace)",
                (long long)M, (long long)K, need, kNoAllocScratchBytes);
  const float* dummy_xs = X;
  bitnet_status st = check_matmul_args("bitnet_i2s_quant_gemv_noalloc", packed, N, K, X, dummy_xs,
                                       M, Y, kMaxTokens);
  if (st != BITNET_OK) return st;
  int dev;
  if ((st = check_device(&dev)) != BITNET_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(dev, &scratch)) != BITNET_OK) return st;
  // The quantizer writes every scratch byte the matmul then reads, so
  // nothing left there by an earlier call is ever used.
  return bitnet_i2s_quant_gemv(packed, N, K, X, M, Y, acc_or_null, scratch,
                               kNoAllocScratchBytes, stream);
}

}  // extern "C"

// ------------------------------------------------------ block-64 formats
namespace {

bitnet_status check_bn(const char* fn, const void* a, const void* b, int64_t N, int64_t K,
                       bool r4) {
  if (a == nullptr || b == nullptr) return fail(BITNET_ERR_INVALID_ARG, "%s: null pointer argument", fn);
  if (N < 1 || K < 64 || K % 64 != 0 || K > kMaxK || (r4 && N % 4 != 0))
    return fail(BITNET_ERR_SHAPE, "%s: N=%lld, K=%lld (K a multiple of 64%s)", fn, (long long)N,
                (long long)K, r4 ? ", N a multiple of 4" : "");
  if (!aligned(a, 16) || !aligned(b, 16))
    return fail(BITNET_ERR_ALIGN, "%s: buffers must be 16-byte aligned", fn);
  return BITNET_OK;
}

int elementwise_grid(int64_t work, int dev) {
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256,
                                                                 int64_t{sm_count(dev)} * 16)));
}

}  // namespace

extern "C" {

size_t bitnet_iq2bn_bytes(int64_t N, int64_t K) {
  if (N < 1 || K < 64 || K % 64 != 0) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K) / 4 + 4 * static_cast<size_t>(N);
}

size_t bitnet_iq1bn_bytes(int64_t N, int64_t K) {
  if (N < 1 || K < 64 || K % 64 != 0) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K / 64) * kIq1BnBlockBytes +
         4 * static_cast<size_t>(N);
}

bitnet_status bitnet_iq2bn_pack(const float* W, int64_t N, int64_t K, int r4, uint8_t* out,
                                void* stream) {
  bitnet_status st = check_bn("bitnet_iq2bn_pack", W, out, N, K, r4 != 0);
  if (st != BITNET_OK) return st;
  int dev;
  if ((st = check_device(&dev)) != BITNET_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* d = reinterpret_cast<float*>(out + N * K / 4);
  bn_row_absmax_kernel<<<static_cast<unsigned>(N), 256, 0, s>>>(W, K, d);
  iq2bn_pack_kernel<<<elementwise_grid(N * K / 16, dev), 256, 0, s>>>(W, N, K, r4 != 0, out, d);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the IQ2_BN pack kernels");
  return ok();
}

bitnet_status bitnet_iq2bn_dequant_f32(const uint8_t* packed, int64_t N, int64_t K, int r4,
                                       float* W_out, void* stream) {
  bitnet_status st = check_bn("bitnet_iq2bn_dequant_f32", packed, W_out, N, K, r4 != 0);
  if (st != BITNET_OK) return st;
  int dev;
  if ((st = check_device(&dev)) != BITNET_OK) return st;
  iq2bn_dequant_kernel<<<elementwise_grid(N * K / 16, dev), 256, 0,
                         static_cast<cudaStream_t>(stream)>>>(
      packed, N, K, r4 != 0, reinterpret_cast<const float*>(packed + N * K / 4), W_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the IQ2_BN dequantize kernel");
  return ok();
}

bitnet_status bitnet_iq1bn_pack(const float* W, int64_t N, int64_t K, uint8_t* out, void* stream) {
  bitnet_status st = check_bn("bitnet_iq1bn_pack", W, out, N, K, false);
  if (st != BITNET_OK) return st;
  int dev;
  if ((st = check_device(&dev)) != BITNET_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t code_bytes = N * (K / 64) * kIq1BnBlockBytes;
  // The fp32 row scales follow the 13-byte blocks, so they are 4-byte
  // aligned only when the number of blocks is a multiple of 4 (it is for
  // every K of the BitNet shapes: K/64 = 40, 108, 128, 448).
  if (code_bytes % 4 != 0)
    return fail(BITNET_ERR_SHAPE, "bitnet_iq1bn_pack: N*(K/64) must be a multiple of 4");
  float* d = reinterpret_cast<float*>(out + code_bytes);
  bn_row_absmax_kernel<<<static_cast<unsigned>(N), 256, 0, s>>>(W, K, d);
  iq1bn_pack_kernel<<<elementwise_grid(code_bytes, dev), 256, 0, s>>>(W, N, K, out, d);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the IQ1_BN pack kernels");
  return ok();
}

bitnet_status bitnet_iq1bn_dequant_f32(const uint8_t* packed, int64_t N, int64_t K, float* W_out,
                                       void* stream) {
  bitnet_status st = check_bn("bitnet_iq1bn_dequant_f32", packed, W_out, N, K, false);
  if (st != BITNET_OK) return st;
  const int64_t code_bytes = N * (K / 64) * kIq1BnBlockBytes;
  if (code_bytes % 4 != 0)
    return fail(BITNET_ERR_SHAPE, "bitnet_iq1bn_dequant_f32: N*(K/64) must be a multiple of 4");
  int dev;
  if ((st = check_device(&dev)) != BITNET_OK) return st;
  iq1bn_dequant_kernel<<<elementwise_grid(code_bytes, dev), 256, 0,
                         static_cast<cudaStream_t>(stream)>>>(
      packed, N, K, reinterpret_cast<const float*>(packed + code_bytes), W_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the IQ1_BN dequantize kernel");
  return ok();
}

bitnet_status bitnet_iq2bn_r4_gemv(const uint8_t* packed, int64_t N, int64_t K, const int8_t* Xq,
                                   const float* xs, int64_t M, float* Y, int32_t* acc_or_null,
                                   void* stream) {
  bitnet_status st = check_bn("bitnet_iq2bn_r4_gemv", packed, Xq, N, K, true);
  if (st != BITNET_OK) return st;
  if (xs == nullptr || Y == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_iq2bn_r4_gemv: null pointer argument");
  if (M < 1 || M > 2 || K > kBnGemvMaxK || N > int64_t{0x7fffffff})
    return fail(BITNET_ERR_SHAPE, "bitnet_iq2bn_r4_gemv: M=%lld (1..2), K=%lld (<= %d)",
                (long long)M, (long long)K, kBnGemvMaxK);
  if (!aligned(Y, 4) || !aligned(xs, 4) || (acc_or_null != nullptr && !aligned(acc_or_null, 4)))
    return fail(BITNET_ERR_ALIGN, "bitnet_iq2bn_r4_gemv: Y, xs and acc must be 4-byte aligned");
  int dev;
  if ((st = check_device(&dev)) != BITNET_OK) return st;
  const int64_t groups = N / 4;
  const int grid = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>((groups + kBnGemvWarps - 1) / kBnGemvWarps, int64_t{sm_count(dev)} * 4)));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 1)
    iq2bn_r4_gemv_kernel<1><<<grid, kBnGemvWarps * 32, 0, s>>>(packed, N, K, Xq, xs, 1, Y,
                                                               acc_or_null);
  else
    iq2bn_r4_gemv_kernel<2><<<grid, kBnGemvWarps * 32, 0, s>>>(packed, N, K, Xq, xs, 2, Y,
                                                               acc_or_null);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the IQ2_BN_R4 matmul kernel");
  return ok();
}

}  // extern "C"

// ------------------------------------------------------------ chains
namespace {

static_assert(sizeof(ChainParamsT<kChainBatch>) <= 32764, "chain kernel parameter block");

// A checked chain: each problem's source and the workspace layout.
//   int32 [0, 64 * count)           finished items per problem, 256 bytes apart
//   int32 [cnt, cnt + sum tiles)    finished slices per row tile
//   int32 [acc, ...)                accumulators, M x N per problem (64-int aligned)
//   ---- zero_bytes: all of the above is zeroed by the call ----
//   fp32  [xs_off, + 2 * count)     activation scales per problem
struct ChainPlan {
  std::vector<int> src;
  std::vector<int64_t> acc_off, cnt_off;
  int64_t launches = 0, done = 0, cnt = 0, acc = 0;
  size_t zero_bytes = 0, xs_off = 0, total_bytes = 0;
};

int64_t align64i(int64_t v) { return (v + 63) & ~int64_t{63}; }

bitnet_status plan_chain(const bitnet_i2s_problem* pr, const int32_t* stage, int count, int64_t M,
                         ChainPlan* plan) {
  const char* fn = "bitnet_i2s_quant_gemv_chain";
  if (pr == nullptr || stage == nullptr || count < 1)
    return fail(BITNET_ERR_INVALID_ARG, "%s: no problems", fn);
  if (count > (1 << 20)) return fail(BITNET_ERR_SHAPE, "%s: %d problems", fn, count);
  if (M < 1 || M > 2)
    return fail(BITNET_ERR_SHAPE, "%s: M=%lld (one or two tokens)", fn, (long long)M);
  for (int i = 0; i < count; ++i) {
    const bitnet_i2s_problem& q = pr[i];
    bitnet_status st = check_matmul_args(fn, q.packed, q.N, q.K, q.X, q.X, M, q.Y, 2);
    if (st != BITNET_OK) return st;
    if (q.acc_or_null != nullptr && !aligned(q.acc_or_null, 4))
      return fail(BITNET_ERR_ALIGN, "%s: acc must be 4-byte aligned", fn);
    const int32_t want = i == 0 ? 0 : stage[i - 1];
    if (stage[i] != want && !(i > 0 && stage[i] == want + 1))
      return fail(BITNET_ERR_INVALID_ARG,
                  "%s: stage[%d]=%d: stages start at 0 and rise by 0 or 1 from problem to problem",
                  fn, i, stage[i]);
  }
  // Outputs must not overlap one another.
  std::vector<std::pair<uintptr_t, uintptr_t>> yr(static_cast<size_t>(count));
  for (int i = 0; i < count; ++i) {
    const uintptr_t b = reinterpret_cast<uintptr_t>(pr[i].Y);
    yr[i] = {b, b + static_cast<uintptr_t>(M * pr[i].N) * sizeof(float)};
  }
  std::sort(yr.begin(), yr.end());
  for (size_t i = 1; i < yr.size(); ++i)
    if (yr[i].first < yr[i - 1].second)
      return fail(BITNET_ERR_INVALID_ARG, "%s: two problems' outputs overlap", fn);
  // An input is either exactly an earlier stage's output (the same pointer,
  // K equal to its N) or memory no output of the chain touches.
  std::unordered_map<uintptr_t, int> by_y;
  for (int i = 0; i < count; ++i) by_y[reinterpret_cast<uintptr_t>(pr[i].Y)] = i;
  plan->src.assign(static_cast<size_t>(count), -1);
  for (int i = 0; i < count; ++i) {
    const uintptr_t xb = reinterpret_cast<uintptr_t>(pr[i].X);
    const auto it = by_y.find(xb);
    if (it != by_y.end()) {
      const int j = it->second;
      if (stage[j] >= stage[i])
        return fail(BITNET_ERR_INVALID_ARG,
                    "%s: problem %d reads the output of problem %d, which is not in an earlier "
                    "stage", fn, i, j);
      if (pr[j].N != pr[i].K)
        return fail(BITNET_ERR_SHAPE, "%s: problem %d has K=%lld but reads an output of N=%lld",
                    fn, i, (long long)pr[i].K, (long long)pr[j].N);
      plan->src[i] = j;
      continue;
    }
    const uintptr_t xe = xb + static_cast<uintptr_t>(M * pr[i].K) * sizeof(float);
    // First output range that ends after the input starts.
    auto hit = std::upper_bound(yr.begin(), yr.end(), std::make_pair(xb, ~uintptr_t{0}));
    if (hit != yr.begin() && std::prev(hit)->second > xb) hit = std::prev(hit);
    if (hit != yr.end() && hit->first < xe)
      return fail(BITNET_ERR_INVALID_ARG,
                  "%s: problem %d's input overlaps an output of the chain without being one", fn,
                  i);
  }
  plan->launches = (count + kChainBatch - 1) / kChainBatch;
  plan->done = 0;
  plan->cnt = int64_t{count} * kChainDoneStride;
  int64_t off = plan->cnt;
  plan->cnt_off.resize(static_cast<size_t>(count));
  for (int i = 0; i < count; ++i) {
    plan->cnt_off[i] = off - plan->cnt;
    off += (pr[i].N + kGemvTileRows - 1) / kGemvTileRows;
  }
  plan->acc = align64i(off);
  off = 0;
  plan->acc_off.resize(static_cast<size_t>(count));
  for (int i = 0; i < count; ++i) {
    plan->acc_off[i] = off;
    off += align64i(M * pr[i].N);
  }
  if (off > int64_t{0x7fffffff})
    return fail(BITNET_ERR_SHAPE, "%s: too many outputs in one chain", fn);
  plan->zero_bytes = align256(static_cast<size_t>(plan->acc + off) * sizeof(int32_t));
  plan->xs_off = plan->zero_bytes;
  plan->total_bytes = plan->xs_off + align256(static_cast<size_t>(count) * 2 * sizeof(float));
  return BITNET_OK;
}

// CTAs of the chain kernel that fit on the device at once.
template <int MT>
bitnet_status chain_grid(int dev, int* out) {
  using C = ChainCfg<MT>;
  static std::atomic<uint8_t> smem_done[kMaxDevices];
  static std::atomic<int> cached[kMaxDevices];
  auto kern = i2s_chain_kernel<MT, kChainBatch>;
  bitnet_status st = ensure_smem(kern, C::kSmemBytes, dev, smem_done);
  if (st != BITNET_OK) return st;
  int v = cached[dev].load(std::memory_order_acquire);
  if (v == 0) {
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::kThreads,
                                                                  C::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "occupancy of the I2_S chain kernel");
    if (per_sm < 1) return fail(BITNET_ERR_UNSUPPORTED, "the chain kernel does not fit on an SM");
    v = std::min(per_sm, C::kCtasPerSm) * sm_count(dev);
    cached[dev].store(v, std::memory_order_release);
  }
  *out = v;
  return BITNET_OK;
}

// A cooperative launch: all of its CTAs are resident at once, which the
// kernel's fixed assignment of items to CTAs needs.
template <int MT>
bitnet_status launch_chain_t(ChainParamsT<kChainBatch>& bp, int grid, cudaStream_t s) {
  using C = ChainCfg<MT>;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(std::min(bp.total_items, grid)));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  std::memset(&attr, 0, sizeof(attr));
  attr.id = cudaLaunchAttributeCooperative;
  attr.val.cooperative = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, i2s_chain_kernel<MT, kChainBatch>, bp);
  if (e != cudaSuccess) return cuda_fail(e, "launch of the I2_S chain kernel");
  return BITNET_OK;
}

// K slices: each stage's problems are cut so that the stage has about as
// many items as the grid has CTAs (at most 16 boxes, 8192 weights, per
// slice); then a zeroing launch and the chain launches, at most kChainBatch
// problems each.  Launches follow one another in stream order, so a problem
// may read the output of one in an earlier launch.
bitnet_status run_chain(const bitnet_i2s_problem* pr, const int32_t* stage, int count, int64_t M,
                        void* workspace, const ChainPlan& plan, cudaStream_t s, int dev) {
  int ctas = 0;
  bitnet_status gst = M == 1 ? chain_grid<1>(dev, &ctas) : chain_grid<2>(dev, &ctas);
  if (gst != BITNET_OK) return gst;
  std::vector<int64_t> stage_tiles(static_cast<size_t>(stage[count - 1]) + 1, 0);
  for (int i = 0; i < count; ++i)
    stage_tiles[stage[i]] += (pr[i].N + kGemvTileRows - 1) / kGemvTileRows;
  int32_t* w = static_cast<int32_t*>(workspace);
  {
    const int64_t n16 = static_cast<int64_t>(plan.zero_bytes / 16);
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(
        std::max<int64_t>(1, std::min<int64_t>((n16 + 255) / 256, 2 * sm_count(dev)))));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaError_t e = cudaLaunchKernelEx(&cfg, chain_zero_kernel, reinterpret_cast<int4*>(w), n16);
    if (e != cudaSuccess) return cuda_fail(e, "launch of the chain zeroing kernel");
  }
  static thread_local ChainParamsT<kChainBatch> bp;  // 28 KB: kept off the stack
  const int64_t nl = plan.launches;
  std::vector<int32_t> splits_of(static_cast<size_t>(count)), items_of(static_cast<size_t>(count));
  for (int64_t c = 0; c < nl; ++c) {
    const int lo = static_cast<int>(count * c / nl);
    const int hi = static_cast<int>(count * (c + 1) / nl);
    bp.count = hi - lo;
    bp.m = static_cast<int32_t>(M);
    bp.done = w + plan.done;
    bp.cnt_base = w + plan.cnt;
    bp.acc_base = w + plan.acc;
    bp.xs_base = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + plan.xs_off);
    int64_t item = 0;
    for (int i = lo; i < hi; ++i) {
      const bitnet_i2s_problem& q = pr[i];
      ChainProblem& P = bp.p[i - lo];
      const int64_t tiles = (q.N + kGemvTileRows - 1) / kGemvTileRows;
      const int64_t nk = (q.K + 511) / 512;
      const int64_t want = std::max<int64_t>(1, ctas / std::max<int64_t>(1, stage_tiles[stage[i]]));
      const int64_t cps = std::min<int64_t>(kChainMaxCps, (nk + std::min(nk, want) - 1) / std::min(nk, want));
      const int64_t splits = (nk + cps - 1) / cps;
      bitnet_status st = encode_u8_2d(&bp.tmap[i - lo], q.packed, static_cast<uint64_t>(q.K / 4),
                                      static_cast<uint64_t>(q.N), 128, kGemvTileRows);
      if (st != BITNET_OK) return st;
      const int j = plan.src[i];
      P.packed = q.packed;
      P.x = j < 0 ? q.X : nullptr;
      P.src_scale = j < 0 ? nullptr
                          : reinterpret_cast<const float*>(pr[j].packed + pr[j].N * (pr[j].K / 4));
      P.y = q.Y;
      P.acc_out = q.acc_or_null;
      P.n = static_cast<int32_t>(q.N);
      P.k = static_cast<int32_t>(q.K);
      P.idx = i;
      P.src = j;
      P.src_splits = j < 0 ? 0 : splits_of[j];
      P.src_cnt = j < 0 ? 0 : static_cast<int32_t>(plan.cnt_off[j]);
      P.src_items = j < 0 ? 0 : items_of[j];
      P.src_acc = j < 0 ? 0 : static_cast<int32_t>(plan.acc_off[j]);
      P.acc = static_cast<int32_t>(plan.acc_off[i]);
      P.cnt = static_cast<int32_t>(plan.cnt_off[i]);
      P.item_start = static_cast<int32_t>(item);
      P.splits = static_cast<int32_t>(splits);
      P.cps = static_cast<int32_t>(cps);
      splits_of[i] = static_cast<int32_t>(splits);
      items_of[i] = static_cast<int32_t>(tiles * splits);
      item += tiles * splits;
      if (item > int64_t{0x7fffffff}) return fail(BITNET_ERR_SHAPE, "chain too large");
    }
    bp.total_items = static_cast<int32_t>(item);
    bp.pad = 0;
    bitnet_status st = M == 1 ? launch_chain_t<1>(bp, ctas, s) : launch_chain_t<2>(bp, ctas, s);
    if (st != BITNET_OK) return st;
  }
  return BITNET_OK;
}

}  // namespace

extern "C" {

size_t bitnet_i2s_quant_gemv_chain_workspace_bytes(const bitnet_i2s_problem* problems,
                                                   const int32_t* stage, int count, int64_t M) {
  ChainPlan plan;
  return plan_chain(problems, stage, count, M, &plan) == BITNET_OK ? plan.total_bytes : 0;
}

bitnet_status bitnet_i2s_quant_gemv_chain(const bitnet_i2s_problem* problems, const int32_t* stage,
                                          int count, int64_t M, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  ChainPlan plan;
  bitnet_status st = plan_chain(problems, stage, count, M, &plan);
  if (st != BITNET_OK) return st;
  if (workspace == nullptr)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_quant_gemv_chain: null workspace");
  if (!aligned(workspace, 256))
    return fail(BITNET_ERR_ALIGN, "bitnet_i2s_quant_gemv_chain: workspace must be 256-byte aligned");
  if (workspace_bytes < plan.total_bytes)
    return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_quant_gemv_chain: workspace of %zu bytes < %zu",
                workspace_bytes, plan.total_bytes);
  int dev;
  if ((st = check_device(&dev)) != BITNET_OK) return st;
  st = run_chain(problems, stage, count, M, workspace, plan, static_cast<cudaStream_t>(stream), dev);
  return st == BITNET_OK ? ok() : st;
}

}  // extern "C"

extern "C" {

bitnet_status bitnet_debug_wait_timeout(int64_t timeout_ns, void* stream) {
  if (timeout_ns < 1000 || timeout_ns > 100000000)
    return fail(BITNET_ERR_INVALID_ARG,
                "bitnet_debug_wait_timeout: timeout_ns must be in [1e3, 1e8]");
  int dev;
  bitnet_status st = check_device(&dev);
  if (st != BITNET_OK) return st;
  stuck_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_ns));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the wait-timeout check");
  return ok();
}

bitnet_status bitnet_device_status(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  unsigned int flags = 0;
  e = cudaMemcpyFromSymbol(&flags, g_error_flags, sizeof(flags));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error flag");
  if (flags != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_error_flags, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error flag");
    return fail(BITNET_ERR_DEVICE_TIMEOUT, "a device-side wait ran out (flags 0x%x)", flags);
  }
  return ok();
}

const char* bitnet_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
