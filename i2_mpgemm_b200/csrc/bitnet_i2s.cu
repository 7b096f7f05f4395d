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
#include <utility>
#include <vector>

#include "bitnet_i2s.h"
#include "gemv_kernel.cuh"
#include "mma_kernel.cuh"
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
// With a work queue, the share of a decode launch's stages in fixed per-CTA
// ranges; the rest is handed out at run time.
constexpr double kStaticShare = 0.7;
bool use_dp4a(int64_t m, int64_t k) {
  return (m >= 1 && m <= 2 && k <= kGemvMaxK) || (m == 1 && k <= kGemvMaxKLong);
}
// K above the short activation slot: the one-token long-K variant.
bool long_k(int64_t k) { return k > kGemvMaxK; }

// Tensor maps, 128-row tiles and their stage counts for every problem.
template <int CAP>
bitnet_status plan_items(BatchParamsT<CAP>& bp) {
  if (bp.queue != nullptr) {
    // Items are handed out in order: the longest ones (largest K) first, so
    // that the last items taken are short and the CTAs end together.
    std::stable_sort(bp.p, bp.p + bp.count,
                     [](const BatchProblem& a, const BatchProblem& b) { return a.k > b.k; });
  }
  int64_t items = 0, stages = 0;
  for (int i = 0; i < bp.count; ++i) {
    BatchProblem& q = bp.p[i];
    bitnet_status st = encode_u8_2d(&bp.tmap[i], q.packed, static_cast<uint64_t>(q.k / 4),
                                    static_cast<uint64_t>(q.n), 128, kGemvTileRows);
    if (st != BITNET_OK) return st;
    q.item_start = static_cast<int32_t>(items);
    q.stage_start = static_cast<int32_t>(stages);
    const int64_t tiles = (q.n + kGemvTileRows - 1) / kGemvTileRows;
    items += tiles;
    stages += tiles * ((q.k + 511) / 512);
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
      const int64_t nk = (q.k + 511) / 512;
      const int64_t tiles = (q.n + kGemvTileRows - 1) / kGemvTileRows;
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
bitnet_status launch_dp4a_t(const BatchParamsT<CAP>& bp, cudaStream_t stream, bool pdl, int dev) {
  using C = GemvCfg<MT, KMAX>;
  static std::atomic<uint8_t> smem_done[kMaxDevices];
  auto kern = i2s_gemv_dp4a_kernel<MT, CAP, KMAX>;
  const int grid = std::min(bp.total_items, C::kCtasPerSm * sm_count(dev));
  bitnet_status st = ensure_smem(kern, C::kSmemBytes, dev, smem_done);
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
template <int CAP>
bitnet_status launch_dp4a(BatchParamsT<CAP>& bp, cudaStream_t stream, bool pdl, int dev,
                          bool wait = true) {
  bitnet_status st = plan_items(bp);
  if (st != BITNET_OK) return st;
  bp.pdl = (pdl && wait) ? 1 : 0;
  int kmax = 0;
  for (int i = 0; i < bp.count; ++i) kmax = std::max(kmax, bp.p[i].k);
  if (bp.m == 1 && long_k(kmax)) return launch_dp4a_t<1, CAP, kGemvMaxKLong>(bp, stream, pdl, dev);
  if (bp.m == 1) return launch_dp4a_t<1, CAP>(bp, stream, pdl, dev);
  return launch_dp4a_t<2, CAP>(bp, stream, pdl, dev);
}

BatchProblem make_problem(const uint8_t* packed, int64_t n, int64_t k, const float* x,
                          const int8_t* xq, const float* xs, float* y, int32_t* acc) {
  BatchProblem q;
  q.packed = packed;
  q.x = x;
  q.xq = const_cast<int8_t*>(xq);
  q.xs = const_cast<float*>(xs);
  q.y = y;
  q.acc = acc;
  q.n = static_cast<int32_t>(n);
  q.k = static_cast<int32_t>(k);
  q.item_start = 0;
  q.stage_start = 0;
  return q;
}

// ------------------------------------------------------ tensor-core path
constexpr int kMmaBatch = 96;  // problems per launch: the parameter block stays under 32 KB

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
    const int64_t n_items = ((q.n + 127) / 128) * token_tiles;
    items += n_items;
    chunks += n_items * ((q.k + 511) / 512);
    if (chunks > int64_t{0x7fffffff}) return fail(BITNET_ERR_SHAPE, "batch too large");
  }
  bp.total_items = static_cast<int32_t>(items);
  bp.total_chunks = static_cast<int32_t>(chunks);
  return BITNET_OK;
}

template <int T, bool kCodes, int CAP>
bitnet_status launch_mma_t(MmaParamsT<CAP>& bp, const int8_t* const* xq, cudaStream_t stream,
                           bool pdl, bool wait, int dev) {
  using C = MmaCfg<T, kCodes>;
  static std::atomic<uint8_t> smem_done[kMaxDevices];
  auto kern = i2s_mma_kernel<T, kCodes, CAP>;
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

// Token tile by M: small tiles with unsigned codes for decode, 128-token
// tiles with signed weights for prefill.
template <int CAP>
bitnet_status launch_mma(MmaParamsT<CAP>& bp, const int8_t* const* xq, cudaStream_t stream,
                         bool pdl, bool wait, int dev) {
  if (bp.m <= 16) return launch_mma_t<16, true>(bp, xq, stream, pdl, wait, dev);
  if (bp.m <= 32) return launch_mma_t<32, true>(bp, xq, stream, pdl, wait, dev);
  if (bp.m <= 64) return launch_mma_t<64, true>(bp, xq, stream, pdl, wait, dev);
  return launch_mma_t<128, false>(bp, xq, stream, pdl, wait, dev);
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
    bp.p[0] = make_problem(packed, n, k, nullptr, xq, xs, y, acc);
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

// Work counters of the decode launches of a batch of `count` problems (the
// two variants are chunked separately, hence at most one launch more).
size_t queue_bytes(int count) {
  return align256(sizeof(int32_t) * static_cast<size_t>((count + kMaxBatch - 1) / kMaxBatch + 1));
}

// Cuts the decode problems (indices into a batch; `nk_of(i)` gives problem
// i's N and K) into launches of at most kMaxBatch problems, in chunks of
// equal size.  A launch runs one kernel variant, chosen by its largest K.
// When the long-K problems have fewer 128-row tiles than the long-K variant
// keeps CTAs on the GPU, every problem joins them in that variant, so the
// launch still has work for every CTA; otherwise the two kinds get separate
// launches.
template <typename NKOf>
std::vector<std::pair<size_t, size_t>> decode_chunks(std::vector<int>& idx, NKOf nk_of, int dev) {
  const auto mid = std::stable_partition(idx.begin(), idx.end(),
                                         [&](int i) { return !long_k(nk_of(i).second); });
  size_t split = static_cast<size_t>(mid - idx.begin());
  int64_t long_tiles = 0;
  for (size_t j = split; j < idx.size(); ++j)
    long_tiles += (nk_of(idx[j]).first + kGemvTileRows - 1) / kGemvTileRows;
  const int64_t long_ctas =
      static_cast<int64_t>(GemvCfg<1, kGemvMaxKLong>::kCtasPerSm) * sm_count(dev);
  if (split < idx.size() && long_tiles < long_ctas) split = 0;  // one group
  std::vector<std::pair<size_t, size_t>> out;
  for (const auto& g : {std::make_pair(size_t{0}, split), std::make_pair(split, idx.size())}) {
    const size_t n = g.second - g.first;
    if (n == 0) continue;
    const size_t nchunks = (n + kMaxBatch - 1) / kMaxBatch;
    for (size_t c = 0; c < nchunks; ++c)
      out.emplace_back(g.first + n * c / nchunks, g.first + n * (c + 1) / nchunks);
  }
  return out;
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
  return align256(static_cast<size_t>(M) * static_cast<size_t>(K)) +
         align256(static_cast<size_t>(M) * sizeof(float));
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
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int8_t* xq = static_cast<int8_t*>(workspace);
  float* xs = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                       align256(static_cast<size_t>(M) * static_cast<size_t>(K)));
  // Quantize with PDL: the kernel waits for whatever precedes it, then lets
  // the matmul launch so its weight loads overlap the quantization.
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(M));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr = pdl_attr(true);
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, act_quant_kernel, X, K, xq, xs);
  if (e != cudaSuccess) return cuda_fail(e, "launch of the activation quant kernel");
  st = run_matmul(packed, N, K, xq, xs, M, Y, acc_or_null, true, s, dev);
  return st == BITNET_OK ? ok() : st;
}

size_t bitnet_i2s_quant_gemv_batched_workspace_bytes(const bitnet_i2s_problem* problems,
                                                     int count, int64_t M) {
  if (problems == nullptr || count < 1 || M < 1) return 0;
  size_t total = 0;
  for (int i = 0; i < count; ++i) {
    const size_t one = bitnet_i2s_quant_gemv_workspace_bytes(M, problems[i].K);
    if (one == 0) return 0;
    total += one;
  }
  return total + queue_bytes(count);
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
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // 1. One launch quantizes every problem's tokens into the workspace.
  // 2. Problems the integer-ALU decode kernel serves (M <= 2, K <= 8192) run
  //    in launches of at most kMaxBatch problems, the rest in launches of at
  //    most kMmaBatch problems on the tensor-core kernel.
  // The first matmul launch waits for the quantizer; every later one is a
  // dependent launch that skips the wait and starts streaming as soon as SMs
  // free up: each launch in the chain starts only after every thread of the
  // one before it has signalled, which the first launch's threads do only
  // after their wait, so all of them start after the quantizer has finished;
  // no matmul writes what another reads; and every CTA waits for the grid
  // before its own before it exits, so the last launch completes last.
  static thread_local QuantBatchParams qp;         // 32 KB: kept off the stack
  static thread_local BatchParamsT<kMaxBatch> bp;  // 30 KB
  std::vector<std::pair<int8_t*, float*>> sl(static_cast<size_t>(count));
  int32_t* queue = nullptr;  // the decode launches' work counters, after the slots
  {
    uint8_t* w = static_cast<uint8_t*>(workspace);
    for (int i = 0; i < count; ++i) {
      sl[i] = {reinterpret_cast<int8_t*>(w),
               reinterpret_cast<float*>(w + align256(static_cast<size_t>(M) * problems[i].K))};
      w += bitnet_i2s_quant_gemv_workspace_bytes(M, problems[i].K);
    }
    queue = reinterpret_cast<int32_t*>(w);
  }
  for (int base = 0; base < count; base += kQuantBatch) {
    const int cnt = std::min(kQuantBatch, count - base);
    qp.count = cnt;
    qp.m = static_cast<int32_t>(M);
    // The first quantizer launch zeroes the counters; every decode launch
    // reads its counter only once the quantizers have finished.
    qp.queue = base == 0 ? queue : nullptr;
    qp.nqueue = base == 0 ? static_cast<int32_t>(queue_bytes(count) / sizeof(int32_t)) : 0;
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
        small, [&](int i) { return std::make_pair(problems[i].N, problems[i].K); }, dev);
    for (size_t c = 0; c < chunks.size(); ++c) {
      const size_t lo = chunks[c].first;
      const size_t hi = chunks[c].second;
      bp.count = static_cast<int32_t>(hi - lo);
      bp.m = static_cast<int32_t>(M);
      bp.queue = queue + c;
      for (size_t i = lo; i < hi; ++i) {
        const bitnet_i2s_problem& q = problems[small[i]];
        bp.p[i - lo] = make_problem(q.packed, q.N, q.K, q.X, sl[small[i]].first,
                                    sl[small[i]].second, q.Y, q.acc_or_null);
      }
      st = launch_dp4a(bp, s, /*pdl=*/true, dev, /*wait=*/first);
      if (st != BITNET_OK) return st;
      first = false;
    }
  }
  if (!big.empty()) {
    // run_mma_batches waits in its first launch only when asked to.
    st = run_mma_batches(big, big_xq, M, /*pdl=*/true, s, dev, /*wait_first=*/first);
    if (st != BITNET_OK) return st;
  }
  return ok();
}

size_t bitnet_i2s_gemv_batched_workspace_bytes(int count) {
  return count < 1 ? 0 : queue_bytes(count);
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
    if (workspace_bytes < queue_bytes(count))
      return fail(BITNET_ERR_INVALID_ARG, "bitnet_i2s_gemv_batched: workspace of %zu bytes < %zu",
                  workspace_bytes, queue_bytes(count));
  }
  int dev;
  bitnet_status st = check_device(&dev);
  if (st != BITNET_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* queue = static_cast<int32_t*>(workspace);
  // Decode-kernel problems in launches of at most kMaxBatch, tensor-core
  // problems in launches of at most kMmaBatch.  The first launch is
  // ordinary, or, with work counters, the one-warp grid that zeroes them
  // after waiting for all earlier work on the stream; either way nothing
  // later starts before that work has finished.  The later launches are
  // dependent launches that start as SMs free up.
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
  bool first = true;
  if (!small.empty()) {
    const auto chunks = decode_chunks(
        small, [&](int i) { return std::make_pair(problems[i].N, problems[i].K); }, dev);
    const size_t nchunks = chunks.size();
    if (queue != nullptr) {
      // A one-warp grid zeroes the counters once the work before this call is
      // done; the first decode launch reads them after waiting for it.
      cudaLaunchConfig_t cfg;
      std::memset(&cfg, 0, sizeof(cfg));
      cfg.gridDim = dim3(1);
      cfg.blockDim = dim3(32);
      cfg.stream = s;
      cudaLaunchAttribute attr = pdl_attr(true);
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      cudaError_t e = cudaLaunchKernelEx(&cfg, zero_counters_kernel, queue,
                                         static_cast<int32_t>(nchunks));
      if (e != cudaSuccess) return cuda_fail(e, "launch of the counter reset");
    }
    for (size_t c = 0; c < nchunks; ++c) {
      const size_t lo = chunks[c].first;
      const size_t hi = chunks[c].second;
      bp.count = static_cast<int32_t>(hi - lo);
      bp.m = static_cast<int32_t>(M);
      bp.queue = queue != nullptr ? queue + c : nullptr;
      for (size_t i = lo; i < hi; ++i) {
        const bitnet_i2s_qproblem& q = problems[small[i]];
        bp.p[i - lo] = make_problem(q.packed, q.N, q.K, nullptr, q.Xq, q.xs, q.Y, q.acc_or_null);
      }
      const bool after_reset = queue != nullptr && c == 0;
      st = launch_dp4a(bp, s, /*pdl=*/!first || after_reset, dev, /*wait=*/after_reset);
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

// Device address of g_noalloc_scratch on the current device, looked up once
// per device.  In host code the array's name is only a host-side stand-in, so
// the address must come from the runtime; it is cached per device id.
bitnet_status noalloc_scratch(int dev, void** out) {
  static std::mutex mu;
  static void* cached[kMaxDevices];
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
    if (p == nullptr) return fail(BITNET_ERR_CUDA, "static scratch has no device address");
    cached[dev] = p;
  }
  *out = cached[dev];
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
