// quant_kernels.cuh -- the memory-bound steps around the matmul: I2_S packing
// of fp32 weights and per-token absmax int8 quantization of activations.
#pragma once

#include "ptx.cuh"

namespace bitnet {

constexpr int kBlockWeights = 128;  // weights per I2_S block
constexpr int kBlockBytes = 32;     // bytes per I2_S block

// Block-wide max of non-negative floats (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ float block_max_nonneg(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = (lane < static_cast<int>(blockDim.x >> 5)) ? red[lane] : 0.0f;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

// ------------------------------------------------------------------ pack
// Step 1: s = max|W| into the scale slot at the packed tensor's tail, which
// the host zeroes first.  For non-negative floats the IEEE bit patterns order
// like the values, so an unsigned atomicMax on the bits is an exact max
// ["How BitNet's 1-Bit (I2_S) Quantization Works ...", Per-Tensor Scaling
// Strategy].
__global__ void __launch_bounds__(256) i2s_absmax_kernel(const float4* __restrict__ w4,
                                                         int64_t n4, unsigned int* scale_bits) {
  __shared__ float red[32];
  float m = 0.0f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(w4 + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  m = block_max_nonneg(m, red);
  if (threadIdx.x == 0 && m > 0.0f) atomicMax(scale_bits, __float_as_uint(m));
}

// Ternary code of one weight: q = clip(round_half_away(w/s), -1, 1), code q+1.
// Because |w/s| <= 1, rounding half away from zero is the pair of comparisons
// t >= 0.5 -> +1 and t <= -0.5 -> -1.
__device__ __forceinline__ uint32_t ternary_code(float w, float s) {
  if (s == 0.0f) return 1u;
  const float t = __fdiv_rn(w, s);
  return t >= 0.5f ? 2u : (t <= -0.5f ? 0u : 1u);
}

// Step 2: each thread writes one 32-bit word, bytes p..p+3 of one block, from
// the 16 weights those bytes hold: offsets 32g + p + i (g = 0..3, i = 0..3)
// inside the block, group g shifted left by 6 - 2g ["How BitNet's 1-Bit
// (I2_S) Quantization Works ...", Ternary Representation and Packing].
__global__ void __launch_bounds__(256) i2s_pack_kernel(const float* __restrict__ w,
                                                       int64_t n_words,
                                                       uint32_t* __restrict__ out,
                                                       const float* __restrict__ scale) {
  const float s = *scale;
  for (int64_t wi = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; wi < n_words;
       wi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t block = wi >> 3;
    const int p = static_cast<int>(wi & 7) * 4;
    const float* base = w + block * kBlockWeights + p;
    uint32_t word = 0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(base + 32 * g));
      const int sh = 6 - 2 * g;
      word |= (ternary_code(v.x, s) << sh) | (ternary_code(v.y, s) << (sh + 8)) |
              (ternary_code(v.z, s) << (sh + 16)) | (ternary_code(v.w, s) << (sh + 24));
    }
    out[wi] = word;
  }
}

// ------------------------------------------------------ activation quant
// One token row: amax over the row, then xq = clamp(rint(x*127/amax))
// ["LLM Quantization Paradigms ...", section 5, The Mathematics of BitNet
// b1.58: per-token AbsMax to 8 bits].  Division and multiplication are the
// IEEE round-to-nearest operations and the rounding to integer is half to
// even, so the codes are a deterministic function of the inputs.  Called by
// every thread of the CTA; k is a multiple of 16.
__device__ __forceinline__ void quantize_row(const float* __restrict__ xrow, int64_t k,
                                             int8_t* __restrict__ qrow, float* __restrict__ xs_out,
                                             float* red) {
  const float4* xr = reinterpret_cast<const float4*>(xrow);
  const int64_t k4 = k >> 2;
  float m = 0.0f;
  for (int64_t i = threadIdx.x; i < k4; i += blockDim.x) {
    const float4 v = xr[i];
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  const float amax = block_max_nonneg(m, red);
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  char4* out = reinterpret_cast<char4*>(qrow);
  for (int64_t i = threadIdx.x; i < k4; i += blockDim.x) {
    const float4 v = xr[i];
    char4 q;
    q.x = static_cast<signed char>(max(-127, min(127, __float2int_rn(__fmul_rn(v.x, inv)))));
    q.y = static_cast<signed char>(max(-127, min(127, __float2int_rn(__fmul_rn(v.y, inv)))));
    q.z = static_cast<signed char>(max(-127, min(127, __float2int_rn(__fmul_rn(v.z, inv)))));
    q.w = static_cast<signed char>(max(-127, min(127, __float2int_rn(__fmul_rn(v.w, inv)))));
    out[i] = q;
  }
  if (threadIdx.x == 0) *xs_out = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
}

// One CTA per token row.  With PDL the kernel first waits for the preceding
// grid, then lets the dependent grid (the matmul) launch and start streaming
// its weights.
__global__ void __launch_bounds__(256) act_quant_kernel(const float* __restrict__ x, int64_t k,
                                                        int8_t* __restrict__ xq,
                                                        float* __restrict__ xs) {
  grid_dependency_wait();
  grid_dependents_launch();
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  quantize_row(x + row * k, k, xq + row * k, xs + row, red);
}

// ------------------------------------------------ dequantize to fp32 (to_float)
// Full-tensor I2_S -> fp32: w_f32 = (code - 1) * s, exact ("ik_llama.cpp 运行
// BitNet b1.58 2B 模型实战", section 5.1: an I2_S tensor is dequantized to f32 in
// full before it is requantized).  One thread per packed 32-bit word writes
// its 16 weights as four float4 (k = 32g + p .. p+3 of the block, g = 0..3).
__global__ void __launch_bounds__(256) i2s_dequant_f32_kernel(const uint32_t* __restrict__ words,
                                                              int64_t n_words,
                                                              const float* __restrict__ scale,
                                                              float* __restrict__ out) {
  const float s = *scale;
  for (int64_t wi = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; wi < n_words;
       wi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t w = __ldg(words + wi);
    float* base = out + (wi >> 3) * kBlockWeights + static_cast<int>(wi & 7) * 4;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int sh = 6 - 2 * g;
      float4 v;
      v.x = __fmul_rn(static_cast<float>(static_cast<int>((w >> sh) & 3u) - 1), s);
      v.y = __fmul_rn(static_cast<float>(static_cast<int>((w >> (sh + 8)) & 3u) - 1), s);
      v.z = __fmul_rn(static_cast<float>(static_cast<int>((w >> (sh + 16)) & 3u) - 1), s);
      v.w = __fmul_rn(static_cast<float>(static_cast<int>((w >> (sh + 24)) & 3u) - 1), s);
      *reinterpret_cast<float4*>(base + 32 * g) = v;
    }
  }
}

// ------------------------------------------------------ AbsMean ternarization
// W~ = RoundClip(W / (gamma + eps), -1, 1), gamma = mean |W| ("LLM
// Quantization Paradigms: FP8, AWQ, EXL2 & BitNet b1.58 in 2026", section 5,
// The Mathematics of BitNet b1.58), the preprocessing step before packing.
// gamma is a deterministic fp64 sum: every CTA adds its grid-stride share in
// a fixed order into partial[blockIdx.x], then one CTA adds the partials in
// index order.  The division and rounding are fp64 (ties away from zero);
// the output is W~ * (float)gamma, which packs losslessly with scale gamma.
constexpr int kAbsMeanBlocks = 1024;

__device__ __forceinline__ double block_sum_f64(double v, double* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = (lane < static_cast<int>(blockDim.x >> 5)) ? red[lane] : 0.0;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

__global__ void __launch_bounds__(256) absmean_partial_kernel(const float* __restrict__ w,
                                                              int64_t count,
                                                              double* __restrict__ partial) {
  __shared__ double red[32];
  double acc = 0.0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    acc += fabs(static_cast<double>(__ldg(w + i)));
  acc = block_sum_f64(acc, red);
  if (threadIdx.x == 0) partial[blockIdx.x] = acc;
}

__global__ void __launch_bounds__(256) absmean_finish_kernel(const double* __restrict__ partial,
                                                             int nparts, int64_t count,
                                                             double* __restrict__ gamma_out) {
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < nparts; ++i) s += partial[i];
    *gamma_out = s / static_cast<double>(count);
  }
}

__global__ void __launch_bounds__(256) ternarize_kernel(const float* __restrict__ w, int64_t count,
                                                        double eps, const double* __restrict__ gamma,
                                                        float* __restrict__ out) {
  const double g = *gamma;
  const double den = g + eps;
  const float gf = static_cast<float>(g);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const double t = static_cast<double>(__ldg(w + i)) / den;
    const double r = fmin(1.0, fmax(-1.0, round(t)));
    out[i] = static_cast<float>(r) * gf;
  }
}

}  // namespace bitnet
