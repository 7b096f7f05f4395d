// bn_kernels.cuh -- the block-64 ternary formats that "ik_llama.cpp 运行 BitNet
// b1.58 2B 模型实战" (sections 5.2, 5.3, 6) converts I2_S into, on the GPU:
// packing fp32 weights into IQ2_BN / IQ2_BN_R4 / IQ1_BN, dequantizing them,
// and a decode matmul on IQ2_BN_R4.
//
// The page fixes 64-weight blocks, one scale per row (each row is quantized
// on its own), IQ2_BN_R4 as IQ2_BN's blocks in groups of 4 rows, and an
// IQ1_BN decode by multiply, add and shift; it leaves the bits inside a
// block open.  The layouts used here:
//   IQ2_BN     block of 64 weights = 16 bytes; weight j in byte j % 16, bits
//              [7-2g : 6-2g] with g = j / 16, code = w + 1.  Row n is K/64
//              blocks; N*K/4 code bytes are followed by N fp32 row scales
//              d_n = max_k |W[n,k]|, and w = clip(round_half_away(W/d_n)).
//   IQ2_BN_R4  N % 4 == 0; block b of row 4G + r at byte
//              ((G*(K/64) + b)*4 + r)*16, so a group of 4 rows is K
//              contiguous bytes in which each block's 4 rows sit together.
//   IQ1_BN     block of 64 weights = 13 bytes: byte i < 12 holds the trits
//              t = w + 1 of weights 5i .. 5i+4, byte 12 those of 60 .. 63 (a
//              fifth trit 0); the byte is ceil(256 v / 243) for
//              v = sum_j t_j 3^(4-j), and trit j is ((byte*3^j) mod 256)*3 >> 8.
//              Row scales as IQ2_BN.
#pragma once

#include "ptx.cuh"
#include "quant_kernels.cuh"

namespace bitnet {

constexpr int kBnBlock = 64;        // weights per block
constexpr int kIq2BnBlockBytes = 16;
constexpr int kIq1BnBlockBytes = 13;

// d_n = max_k |W[n,k]|, one CTA per row (blockDim 256).
__global__ void __launch_bounds__(256) bn_row_absmax_kernel(const float* __restrict__ w,
                                                            int64_t k, float* __restrict__ d) {
  __shared__ float red[32];
  const float4* row = reinterpret_cast<const float4*>(w + blockIdx.x * k);
  float m = 0.0f;
  for (int64_t i = threadIdx.x; i < k / 4; i += blockDim.x) {
    const float4 v = __ldg(row + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  m = block_max_nonneg(m, red);
  if (threadIdx.x == 0) d[blockIdx.x] = m;
}

// Byte offset of block b of row n in IQ2_BN (r4 = false) or IQ2_BN_R4.
__device__ __forceinline__ int64_t iq2bn_block_offset(int64_t n, int64_t b, int64_t nb, bool r4) {
  return r4 ? (((n >> 2) * nb + b) * 4 + (n & 3)) * kIq2BnBlockBytes
            : (n * nb + b) * kIq2BnBlockBytes;
}

// Codes: each thread writes one 32-bit word, bytes p..p+3 of one block,
// from the 16 weights they hold (offsets 16g + p + i of the block).
__global__ void __launch_bounds__(256) iq2bn_pack_kernel(const float* __restrict__ w, int64_t n_rows,
                                                         int64_t k, bool r4, uint8_t* __restrict__ out,
                                                         const float* __restrict__ d) {
  const int64_t nb = k / kBnBlock;
  const int64_t words = n_rows * nb * 4;
  for (int64_t wi = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; wi < words;
       wi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t blk = wi >> 2;
    const int p = static_cast<int>(wi & 3) * 4;
    const int64_t n = blk / nb, b = blk - n * nb;
    const float s = d[n];
    const float* base = w + n * k + b * kBnBlock + p;
    uint32_t word = 0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(base + 16 * g));
      const int sh = 6 - 2 * g;
      word |= (ternary_code(v.x, s) << sh) | (ternary_code(v.y, s) << (sh + 8)) |
              (ternary_code(v.z, s) << (sh + 16)) | (ternary_code(v.w, s) << (sh + 24));
    }
    *reinterpret_cast<uint32_t*>(out + iq2bn_block_offset(n, b, nb, r4) + p) = word;
  }
}

// IQ2_BN / IQ2_BN_R4 -> fp32, one word (16 weights) per thread.
__global__ void __launch_bounds__(256) iq2bn_dequant_kernel(const uint8_t* __restrict__ in,
                                                            int64_t n_rows, int64_t k, bool r4,
                                                            const float* __restrict__ d,
                                                            float* __restrict__ w) {
  const int64_t nb = k / kBnBlock;
  const int64_t words = n_rows * nb * 4;
  for (int64_t wi = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; wi < words;
       wi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t blk = wi >> 2;
    const int p = static_cast<int>(wi & 3) * 4;
    const int64_t n = blk / nb, b = blk - n * nb;
    const float s = d[n];
    const uint32_t word = __ldg(reinterpret_cast<const uint32_t*>(in + iq2bn_block_offset(n, b, nb, r4) + p));
    float* base = w + n * k + b * kBnBlock + p;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int sh = 6 - 2 * g;
      float4 v;
      v.x = static_cast<float>(static_cast<int>((word >> sh) & 3u) - 1) * s;
      v.y = static_cast<float>(static_cast<int>((word >> (sh + 8)) & 3u) - 1) * s;
      v.z = static_cast<float>(static_cast<int>((word >> (sh + 16)) & 3u) - 1) * s;
      v.w = static_cast<float>(static_cast<int>((word >> (sh + 24)) & 3u) - 1) * s;
      *reinterpret_cast<float4*>(base + 16 * g) = v;
    }
  }
}

// IQ1_BN: one byte (5 or 4 weights) per thread.
__global__ void __launch_bounds__(256) iq1bn_pack_kernel(const float* __restrict__ w, int64_t n_rows,
                                                         int64_t k, uint8_t* __restrict__ out,
                                                         const float* __restrict__ d) {
  const int64_t nb = k / kBnBlock;
  const int64_t bytes = n_rows * nb * kIq1BnBlockBytes;
  for (int64_t bi = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; bi < bytes;
       bi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t blk = bi / kIq1BnBlockBytes;
    const int i = static_cast<int>(bi - blk * kIq1BnBlockBytes);
    const int64_t n = blk / nb, b = blk - n * nb;
    const float s = d[n];
    const float* base = w + n * k + b * kBnBlock;
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      const int e = 5 * i + j;
      const uint32_t t = e < kBnBlock ? ternary_code(__ldg(base + e), s) : 0u;
      v = 3u * v + t;
    }
    out[bi] = static_cast<uint8_t>((256u * v + 242u) / 243u);  // ceil(256 v / 243)
  }
}

// IQ1_BN -> fp32, one byte per thread: trit j = ((q * 3^j) mod 256) * 3 >> 8.
__global__ void __launch_bounds__(256) iq1bn_dequant_kernel(const uint8_t* __restrict__ in,
                                                            int64_t n_rows, int64_t k,
                                                            const float* __restrict__ d,
                                                            float* __restrict__ w) {
  const int64_t nb = k / kBnBlock;
  const int64_t bytes = n_rows * nb * kIq1BnBlockBytes;
  for (int64_t bi = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; bi < bytes;
       bi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t blk = bi / kIq1BnBlockBytes;
    const int i = static_cast<int>(bi - blk * kIq1BnBlockBytes);
    const int64_t n = blk / nb, b = blk - n * nb;
    const float s = d[n];
    const uint32_t q = __ldg(in + bi);
    float* base = w + n * k + b * kBnBlock;
    uint32_t p3 = 1;
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      const int e = 5 * i + j;
      const int t = static_cast<int>((((q * p3) & 255u) * 3u) >> 8);
      if (e < kBnBlock) base[e] = static_cast<float>(t - 1) * s;
      p3 *= 3u;
    }
  }
}

// ------------------------------------------------------ IQ2_BN_R4 decode matmul
// One warp per group of 4 rows.  The group is K contiguous bytes, block b
// holding the 4 rows' 16 bytes next to each other; lane l takes blocks l,
// l + 32, ... and reads each one's 64 bytes with four 16-byte loads (a warp
// reads 2 KB in a row), so every activation word it loads from shared
// memory serves 4 rows.  Codes are used without shifts: word &
// (3 << (6-2g)) is code * 4^(3-g) in every byte, accumulated per group with
// dp4a and rescaled exactly at the end; sum_k x is subtracted because
// w = code - 1.  Then y = ((float)acc * xs[m]) * d_n.
constexpr int kBnGemvWarps = 8;
constexpr int kBnGemvMaxK = 8192;

template <int MT>
__global__ void __launch_bounds__(kBnGemvWarps * 32) iq2bn_r4_gemv_kernel(
    const uint8_t* __restrict__ r4, int64_t n_rows, int64_t k, const int8_t* __restrict__ xq,
    const float* __restrict__ xs, int m_tokens, float* __restrict__ y, int32_t* __restrict__ acc) {
  __shared__ __align__(16) int8_t xsm[MT * kBnGemvMaxK];
  __shared__ int xsum_sm[MT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* __restrict__ d = reinterpret_cast<const float*>(r4 + n_rows * (k >> 2));
  // Stage the activations (M x K int8) and their sums.
  for (int64_t i = threadIdx.x; i < static_cast<int64_t>(m_tokens) * k / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(xsm)[i] = __ldg(reinterpret_cast<const uint4*>(xq) + i);
  __syncthreads();
  if (warp < m_tokens) {
    int s = 0;
    for (int64_t off = lane * 16; off < k; off += 512) {
      const uint4 v = *reinterpret_cast<const uint4*>(xsm + warp * k + off);
      s = __dp4a(static_cast<int>(v.x), 0x01010101, s);
      s = __dp4a(static_cast<int>(v.y), 0x01010101, s);
      s = __dp4a(static_cast<int>(v.z), 0x01010101, s);
      s = __dp4a(static_cast<int>(v.w), 0x01010101, s);
    }
    s = __reduce_add_sync(0xffffffffu, s);
    if (lane == 0) xsum_sm[warp] = s;
  }
  __syncthreads();
  const int64_t nb = k / kBnBlock;
  const int64_t groups = n_rows >> 2;
  for (int64_t grp = static_cast<int64_t>(blockIdx.x) * kBnGemvWarps + warp; grp < groups;
       grp += static_cast<int64_t>(gridDim.x) * kBnGemvWarps) {
    const uint4* base = reinterpret_cast<const uint4*>(r4 + grp * k);  // 4 uint4 per block
    int a[4][MT][4];  // [row][token][group]
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int g = 0; g < 4; ++g) a[r][m][g] = 0;
    for (int64_t b = lane; b < nb; b += 32) {
      uint4 wv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) wv[r] = __ldcs(base + b * 4 + r);  // read once: evict first
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4* xb = reinterpret_cast<const uint4*>(xsm + m * k + b * kBnBlock);
        uint4 xv[4];  // xv[g]: activations 16g .. 16g+15 of the block
#pragma unroll
        for (int g = 0; g < 4; ++g) xv[g] = xb[g];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint32_t ww[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint32_t mask = 0x03030303u << (6 - 2 * g);
            const uint32_t xx[4] = {xv[g].x, xv[g].y, xv[g].z, xv[g].w};
            int s = a[r][m][g];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              int d4;
              asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d4) : "r"(ww[i] & mask), "r"(xx[i]), "r"(s));
              s = d4;
            }
            a[r][m][g] = s;
          }
        }
      }
    }
    // Rescale the groups (exact multiples of 4^(3-g)), add over the lanes.
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int64_t n = grp * 4 + r;
      const float dn = __ldg(d + n);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        int part = (a[r][m][0] >> 6) + (a[r][m][1] >> 4) + (a[r][m][2] >> 2) + a[r][m][3];
        part = __reduce_add_sync(0xffffffffu, part);
        if (lane == 0 && m < m_tokens) {
          const int dot = part - xsum_sm[m];
          y[m * n_rows + n] = __fmul_rn(__fmul_rn(__int2float_rn(dot), __ldg(xs + m)), dn);
          if (acc != nullptr) acc[m * n_rows + n] = dot;
        }
      }
    }
  }
}

}  // namespace bitnet
