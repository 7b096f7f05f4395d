/*
 * i2s_oracle.c -- plain scalar C oracle for the I2_S ternary x int8 matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's shared library.  No
 * product code path may call it, and it shares no code, header, table or
 * helper with the CUDA library under i2_mpgemm_b200/csrc.
 *
 * Every function is the plain definition of one step, written as loops in
 * the order the steps are described, with no blocking, fusion or reordering.
 * Build flags: -O2 -ffp-contract=off -fno-fast-math (no FMA contraction, IEEE
 * fp32 divide and multiply, default round-to-nearest-even mode).
 *
 * Sources (web pages; cited by title and section):
 *   [P1] "How BitNet's 1-Bit (I2_S) Quantization Works Compared to Standard
 *        LLM Quantization" (instagit deep-dive on microsoft/BitNet).
 *   [P2] "BitNet Inference Preprocessing: Converting Hugging Face Checkpoints
 *        to I2S GGUF".
 *   [P3] "ik_llama.cpp 运行 BitNet b1.58 2B 模型实战：从 bitnet-b1.58 架构兼容到
 *        I2_S 量化转换".
 *   [P5] "LLM Quantization Paradigms: FP8, AWQ, EXL2 & BitNet b1.58 in 2026".
 *
 * Readings taken where the pages are silent or garbled (each is also listed
 * in the design notes):
 *   R1  Four 2-bit codes per byte.  [P1 §Ternary Representation and Packing]
 *       says both "2 bits per weight" and "32 values into a byte"; only the
 *       first is consistent with the shift amount 6-2*group_idx (four groups).
 *   R2  Block of 128 weights -> 32 bytes.  Weight j of a block (j = 0..127)
 *       sits in byte j%32 of the block, group g = j/32, bits [7-2g : 6-2g].
 *       The block is taken over the row-major flattened index n*K+k; K must
 *       be a multiple of 128 so a block never straddles two rows.
 *   R3  Code = w + 1 for w in {-1,0,+1} [P1 §Ternary Representation and
 *       Packing]; code 3 is never written and is an error on unpack.
 *   R4  Float -> ternary before packing: t = w / s (fp32 IEEE divide) with
 *       s = max|w|; q = clip(round_half_away(t), -1, 1).  The pages only say
 *       the packing is lossless for already-ternary input [P2 §The Two-Stage
 *       BitNet Inference Preprocessing Pipeline]; this rule is lossless there.
 *   R5  The fp32 scale s = max|w| [P1 §Per-Tensor Scaling Strategy] is stored
 *       little-endian right after the N*K/4 code bytes; total N*K/4 + 4 bytes.
 *       An all-zero tensor stores s = 0 and code 1 everywhere.
 *   R6  Per-token absmax int8 activations [P5 §5, "The Mathematics of BitNet
 *       b1.58"]: amax = max_k |x|; inv = 127/amax (fp32 divide);
 *       xq = clamp(round_half_even(x*inv), -127, 127); xs = amax/127 (fp32
 *       divide).  A zero row gives xq = 0 and xs = 0.
 *   R7  Contraction [P5 §5 figure "BitNet b1.58 Ternary Matrix
 *       Multiplication"]: acc = sum_k w*xq in int32 (add when w = +1,
 *       subtract when w = -1, skip when w = 0).
 *   R8  Dequant [P1 §How I2_S Kernels Process the Format, multiply by the
 *       shared per-tensor scale]: y = ((float)acc * xs[m]) * s, two separately
 *       rounded fp32 multiplies in that order.
 *   R9  AbsMean ternarization [P5 §5, "The Mathematics of BitNet b1.58"]:
 *       gamma = mean |W| (fp64 sum in index order); W~ = RoundClip(W /
 *       (gamma + eps), -1, 1) in fp64 with round half away from zero; the
 *       tensor handed to pack is W~ * (float)gamma.
 *   R10 Dequantize to fp32 [P3 §5.1, full-tensor to_float before
 *       requantizing]: w_f32 = (float)w * s, exact.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define I2S_BLOCK 128 /* weights per block (R2) */
#define I2S_BLOCK_BYTES 32 /* bytes per block */

/* Status codes (the oracle's own; unrelated to the library's). */
#define ORC_OK 0
#define ORC_BAD_SHAPE -1
#define ORC_BAD_CODE -2
#define ORC_BAD_ARG -3

static int shape_ok(int64_t n, int64_t k) {
  return n >= 1 && k >= 1 && (k % I2S_BLOCK) == 0;
}

/* Number of bytes of a packed tensor: 2 bits per weight plus the fp32 scale (R5). */
size_t i2s_oracle_packed_bytes(int64_t n, int64_t k) {
  return (size_t)(n * k / 4) + 4;
}

/* Where weight (n, k) lives: byte index and left shift (R2). */
static void locate(int64_t k_dim, int64_t n, int64_t k, int64_t* byte_index, int* shift) {
  int64_t e = n * k_dim + k;          /* flattened row-major index */
  int64_t block = e / I2S_BLOCK;
  int64_t j = e % I2S_BLOCK;          /* position inside the block */
  int64_t group = j / 32;             /* 0..3 */
  int64_t pos = j % 32;               /* byte inside the block */
  *byte_index = block * I2S_BLOCK_BYTES + pos;
  *shift = 6 - 2 * (int)group;
}

/* Per-tensor scale s = max |w| (R5). */
static float absmax_f32(const float* w, int64_t count) {
  float s = 0.0f;
  for (int64_t i = 0; i < count; ++i) {
    float a = fabsf(w[i]);
    if (a > s) s = a;
  }
  return s;
}

/* Round half away from zero, then clip to [-1, 1] (R4). */
static int ternary_of(float w, float s) {
  if (s == 0.0f) return 0;
  float t = w / s;
  float r = roundf(t);
  if (r > 1.0f) r = 1.0f;
  if (r < -1.0f) r = -1.0f;
  return (int)r;
}

/* Pack fp32 weights W[N,K] (row-major) into I2_S: codes then scale (R1-R5). */
int i2s_oracle_pack(const float* w, int64_t n, int64_t k, uint8_t* packed) {
  if (!w || !packed) return ORC_BAD_ARG;
  if (!shape_ok(n, k)) return ORC_BAD_SHAPE;
  int64_t code_bytes = n * k / 4;
  memset(packed, 0, (size_t)code_bytes);
  float s = absmax_f32(w, n * k);
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t c = 0; c < k; ++c) {
      int q = ternary_of(w[r * k + c], s);
      int code = q + 1; /* R3 */
      int64_t bi;
      int sh;
      locate(k, r, c, &bi, &sh);
      packed[bi] = (uint8_t)(packed[bi] | (code << sh));
    }
  }
  memcpy(packed + code_bytes, &s, sizeof(float)); /* little-endian host */
  return ORC_OK;
}

/* The stored per-tensor scale (R5). */
float i2s_oracle_scale(const uint8_t* packed, int64_t n, int64_t k) {
  float s;
  memcpy(&s, packed + n * k / 4, sizeof(float));
  return s;
}

/* One weight w in {-1,0,+1} read back from the packed bytes (R2, R3).
 * Returns 2 (impossible weight) when the stored code is 3. */
static int weight_at(const uint8_t* packed, int64_t k_dim, int64_t n, int64_t k) {
  int64_t bi;
  int sh;
  locate(k_dim, n, k, &bi, &sh);
  int code = (packed[bi] >> sh) & 3;
  if (code == 3) return 2;
  return code - 1;
}

/* Unpack to int8 T[N,K] in {-1,0,+1} plus the scale. */
int i2s_oracle_unpack(const uint8_t* packed, int64_t n, int64_t k, int8_t* t, float* scale) {
  if (!packed || !t) return ORC_BAD_ARG;
  if (!shape_ok(n, k)) return ORC_BAD_SHAPE;
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t c = 0; c < k; ++c) {
      int v = weight_at(packed, k, r, c);
      if (v == 2) return ORC_BAD_CODE;
      t[r * k + c] = (int8_t)v;
    }
  }
  if (scale) *scale = i2s_oracle_scale(packed, n, k);
  return ORC_OK;
}

/* Per-token absmax int8 quantization of X[M,K] (R6). */
int i2s_oracle_act_quant(const float* x, int64_t m, int64_t k, int8_t* xq, float* xs) {
  if (!x || !xq || !xs) return ORC_BAD_ARG;
  if (m < 1 || k < 1) return ORC_BAD_SHAPE;
  for (int64_t r = 0; r < m; ++r) {
    const float* row = x + r * k;
    float amax = 0.0f;
    for (int64_t c = 0; c < k; ++c) {
      float a = fabsf(row[c]);
      if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
      for (int64_t c = 0; c < k; ++c) xq[r * k + c] = 0;
      xs[r] = 0.0f;
      continue;
    }
    float inv = 127.0f / amax;
    for (int64_t c = 0; c < k; ++c) {
      float v = nearbyintf(row[c] * inv); /* round half to even */
      if (v > 127.0f) v = 127.0f;
      if (v < -127.0f) v = -127.0f;
      xq[r * k + c] = (int8_t)v;
    }
    xs[r] = amax / 127.0f;
  }
  return ORC_OK;
}

/* One output element: exact int32 dot product (R7) and the dequant (R8). */
static int one_output(const uint8_t* packed, int64_t k_dim, int64_t n, const int8_t* xq_row,
                      float xs_m, float s, float* y, int32_t* acc) {
  int32_t a = 0;
  for (int64_t c = 0; c < k_dim; ++c) {
    int w = weight_at(packed, k_dim, n, c);
    if (w == 2) return ORC_BAD_CODE;
    if (w == 1) a += (int32_t)xq_row[c];
    else if (w == -1) a -= (int32_t)xq_row[c];
  }
  if (acc) *acc = a;
  if (y) {
    float t = (float)a * xs_m;
    *y = t * s;
  }
  return ORC_OK;
}

/* Y[M,N] = dequant(Xq[M,K] . T[N,K]^T) for every output (R7, R8). */
int i2s_oracle_gemm(const uint8_t* packed, int64_t n, int64_t k, const int8_t* xq,
                    const float* xs, int64_t m, float* y, int32_t* acc) {
  if (!packed || !xq || !xs) return ORC_BAD_ARG;
  if (!shape_ok(n, k) || m < 1) return ORC_BAD_SHAPE;
  float s = i2s_oracle_scale(packed, n, k);
  for (int64_t r = 0; r < m; ++r) {
    for (int64_t c = 0; c < n; ++c) {
      int st = one_output(packed, k, c, xq + r * k, xs[r], s, y ? &y[r * n + c] : 0,
                          acc ? &acc[r * n + c] : 0);
      if (st != ORC_OK) return st;
    }
  }
  return ORC_OK;
}

/* The same, for a list of (token, row) output positions only. */
int i2s_oracle_gemm_sampled(const uint8_t* packed, int64_t n, int64_t k, const int8_t* xq,
                            const float* xs, int64_t m, const int64_t* pos_m,
                            const int64_t* pos_n, int64_t count, float* y, int32_t* acc) {
  if (!packed || !xq || !xs || !pos_m || !pos_n) return ORC_BAD_ARG;
  if (!shape_ok(n, k) || m < 1 || count < 0) return ORC_BAD_SHAPE;
  float s = i2s_oracle_scale(packed, n, k);
  for (int64_t i = 0; i < count; ++i) {
    int64_t r = pos_m[i], c = pos_n[i];
    if (r < 0 || r >= m || c < 0 || c >= n) return ORC_BAD_ARG;
    int st = one_output(packed, k, c, xq + r * k, xs[r], s, y ? &y[i] : 0, acc ? &acc[i] : 0);
    if (st != ORC_OK) return st;
  }
  return ORC_OK;
}

/* Activation quantization followed by the matmul (R6 then R7, R8).
 * xq_out / xs_out may be NULL; scratch for them is taken from the heap. */
int i2s_oracle_quant_gemm(const uint8_t* packed, int64_t n, int64_t k, const float* x,
                          int64_t m, float* y, int32_t* acc, int8_t* xq_out, float* xs_out) {
  if (!packed || !x) return ORC_BAD_ARG;
  if (!shape_ok(n, k) || m < 1) return ORC_BAD_SHAPE;
  int8_t* xq = xq_out ? xq_out : (int8_t*)malloc((size_t)(m * k));
  float* xs = xs_out ? xs_out : (float*)malloc((size_t)m * sizeof(float));
  int st = (xq && xs) ? ORC_OK : ORC_BAD_ARG;
  if (st == ORC_OK) st = i2s_oracle_act_quant(x, m, k, xq, xs);
  if (st == ORC_OK) st = i2s_oracle_gemm(packed, n, k, xq, xs, m, y, acc);
  if (!xq_out) free(xq);
  if (!xs_out) free(xs);
  return st;
}

/* AbsMean ternarization (R9).  w_out receives W~ * (float)gamma. */
int i2s_oracle_ternarize_absmean(const float* w, int64_t count, double eps, float* w_out,
                                 double* gamma_out) {
  if (!w || !w_out || count < 1) return ORC_BAD_ARG;
  double sum = 0.0;
  for (int64_t i = 0; i < count; ++i) sum += fabs((double)w[i]);
  double gamma = sum / (double)count;
  float gamma_f = (float)gamma;
  for (int64_t i = 0; i < count; ++i) {
    double t = (double)w[i] / (gamma + eps);
    double r = round(t);
    if (r > 1.0) r = 1.0;
    if (r < -1.0) r = -1.0;
    w_out[i] = (float)r * gamma_f;
  }
  if (gamma_out) *gamma_out = gamma;
  return ORC_OK;
}

/* Full-tensor dequantization to fp32 (R10). */
int i2s_oracle_dequant_f32(const uint8_t* packed, int64_t n, int64_t k, float* w_out) {
  if (!packed || !w_out) return ORC_BAD_ARG;
  if (!shape_ok(n, k)) return ORC_BAD_SHAPE;
  float s = i2s_oracle_scale(packed, n, k);
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t c = 0; c < k; ++c) {
      int v = weight_at(packed, k, r, c);
      if (v == 2) return ORC_BAD_CODE;
      w_out[r * k + c] = (float)v * s;
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------
 * The block-64 formats that "ik_llama.cpp 运行 BitNet b1.58 2B 模型实战" (§5.2,
 * §5.3, §6) converts I2_S into: IQ2_BN (about 2 bits per weight), its 4-row
 * interleaved variant IQ2_BN_R4, and IQ1_BN (1.625 bits per weight).  The
 * page fixes the block of 64 weights (K must be a multiple of 64), the bit
 * rates, the conversion chain I2_S -> f32 -> IQ2_BN (§5.1), that each row is
 * quantized on its own, that R4 packs rows in groups of 4 with IQ2_BN's block
 * structure, and that IQ1_BN is decoded with multiplies, adds and shifts.  It
 * elides the bits inside a block, so the layouts below are readings, and
 * their byte-level parity is unpinned by anything outside this file:
 *   R11 IQ2_BN: a block of 64 weights is 16 bytes; weight j of the block sits
 *       in byte j % 16, group g = j / 16, bits [7-2g : 6-2g], code = q + 1
 *       (the I2_S grouping of R2 on 64-weight blocks).  Row n is K/64 blocks;
 *       the tensor is N*K/4 code bytes followed by N fp32 row scales
 *       d_n = max_k |W[n,k]|, and q = clip(round_half_away(W/d_n), -1, 1) as
 *       in R4 with the row's scale (d_n = 0 gives code 1).
 *   R12 IQ2_BN_R4: N a multiple of 4; block b of row 4G + r is stored at byte
 *       ((G * (K/64) + b) * 4 + r) * 16, so the four rows' blocks b sit next
 *       to each other; codes inside a block and the N row scales as R11.
 *   R13 IQ1_BN: a block of 64 weights is 13 bytes: byte i < 12 holds the
 *       trits t = q + 1 of weights 5i .. 5i+4, byte 12 those of weights
 *       60 .. 63 (a fifth trit 0).  With v = sum_j t_j 3^(4-j) (the first
 *       weight most significant) the byte stores ceil(256 v / 243); trit j is
 *       ((byte * 3^j) mod 256) * 3 >> 8.  Row scales as R11.
 *   R14 The matmul on these formats is R7 with the row's scale in place of
 *       the tensor's: y = ((float)acc * xs[m]) * d_n.
 */
#define BN_BLOCK 64
#define IQ2BN_BLOCK_BYTES 16
#define IQ1BN_BLOCK_BYTES 13

static int bn_shape_ok(int64_t n, int64_t k) { return n >= 1 && k >= 1 && k % BN_BLOCK == 0; }

size_t i2s_oracle_iq2bn_bytes(int64_t n, int64_t k) { return (size_t)(n * k / 4 + 4 * n); }
size_t i2s_oracle_iq1bn_bytes(int64_t n, int64_t k) {
  return (size_t)(n * (k / BN_BLOCK) * IQ1BN_BLOCK_BYTES + 4 * n);
}

/* Row scales d_n = max_k |W[n,k]| (R11). */
static void row_absmax(const float* w, int64_t n, int64_t k, float* d) {
  for (int64_t r = 0; r < n; ++r) d[r] = absmax_f32(w + r * k, k);
}

/* Byte index and shift of weight (n, c) in IQ2_BN (R11) or IQ2_BN_R4 (R12). */
static void iq2bn_locate(int64_t k_dim, int64_t n, int64_t c, int r4, int64_t* byte_index,
                         int* shift) {
  int64_t b = c / BN_BLOCK, j = c % BN_BLOCK;
  int64_t nb = k_dim / BN_BLOCK;
  int64_t block_base;
  if (r4) block_base = (((n / 4) * nb + b) * 4 + (n % 4)) * IQ2BN_BLOCK_BYTES;
  else block_base = (n * nb + b) * IQ2BN_BLOCK_BYTES;
  *byte_index = block_base + j % IQ2BN_BLOCK_BYTES;
  *shift = 6 - 2 * (int)(j / IQ2BN_BLOCK_BYTES);
}

/* Pack fp32 W[N,K] into IQ2_BN (r4 = 0) or IQ2_BN_R4 (r4 = 1). */
int i2s_oracle_iq2bn_pack(const float* w, int64_t n, int64_t k, int r4, uint8_t* out) {
  if (!w || !out) return ORC_BAD_ARG;
  if (!bn_shape_ok(n, k) || (r4 && n % 4 != 0)) return ORC_BAD_SHAPE;
  int64_t code_bytes = n * k / 4;
  memset(out, 0, (size_t)code_bytes);
  float* d = (float*)(out + code_bytes); /* 4-byte aligned when out is */
  float* dtmp = (float*)malloc((size_t)n * sizeof(float));
  if (!dtmp) return ORC_BAD_ARG;
  row_absmax(w, n, k, dtmp);
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t c = 0; c < k; ++c) {
      int code = ternary_of(w[r * k + c], dtmp[r]) + 1;
      int64_t bi;
      int sh;
      iq2bn_locate(k, r, c, r4, &bi, &sh);
      out[bi] = (uint8_t)(out[bi] | (code << sh));
    }
  }
  memcpy(d, dtmp, (size_t)n * sizeof(float));
  free(dtmp);
  return ORC_OK;
}

/* IQ2_BN or IQ2_BN_R4 -> int8 T[N,K] and the row scales d[N]. */
int i2s_oracle_iq2bn_unpack(const uint8_t* p, int64_t n, int64_t k, int r4, int8_t* t, float* d) {
  if (!p || !t) return ORC_BAD_ARG;
  if (!bn_shape_ok(n, k) || (r4 && n % 4 != 0)) return ORC_BAD_SHAPE;
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t c = 0; c < k; ++c) {
      int64_t bi;
      int sh;
      iq2bn_locate(k, r, c, r4, &bi, &sh);
      int code = (p[bi] >> sh) & 3;
      if (code == 3) return ORC_BAD_CODE;
      t[r * k + c] = (int8_t)(code - 1);
    }
  }
  if (d) memcpy(d, p + n * k / 4, (size_t)n * sizeof(float));
  return ORC_OK;
}

/* The IQ1_BN byte of five trits t[0..4] (R13). */
static uint8_t iq1bn_encode(const int* t) {
  int v = 0;
  for (int j = 0; j < 5; ++j) v = 3 * v + t[j];
  return (uint8_t)((256 * v + 242) / 243); /* ceil(256 v / 243) */
}

/* Trit j (0..4) of an IQ1_BN byte (R13). */
static int iq1bn_trit(uint8_t q, int j) {
  int p3 = 1;
  for (int i = 0; i < j; ++i) p3 *= 3;
  return ((((int)q * p3) & 255) * 3) >> 8;
}

int i2s_oracle_iq1bn_encode_byte(const int* trits) { return iq1bn_encode(trits); }
int i2s_oracle_iq1bn_trit(int byte, int j) { return iq1bn_trit((uint8_t)byte, j); }

/* Pack fp32 W[N,K] into IQ1_BN (R13). */
int i2s_oracle_iq1bn_pack(const float* w, int64_t n, int64_t k, uint8_t* out) {
  if (!w || !out) return ORC_BAD_ARG;
  if (!bn_shape_ok(n, k)) return ORC_BAD_SHAPE;
  int64_t nb = k / BN_BLOCK;
  int64_t code_bytes = n * nb * IQ1BN_BLOCK_BYTES;
  float* d = (float*)malloc((size_t)n * sizeof(float));
  if (!d) return ORC_BAD_ARG;
  row_absmax(w, n, k, d);
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      uint8_t* blk = out + (r * nb + b) * IQ1BN_BLOCK_BYTES;
      for (int i = 0; i < IQ1BN_BLOCK_BYTES; ++i) {
        int t[5] = {0, 0, 0, 0, 0};
        for (int j = 0; j < 5; ++j) {
          int e = 5 * i + j; /* weight of the block */
          if (e < BN_BLOCK) t[j] = ternary_of(w[r * k + b * BN_BLOCK + e], d[r]) + 1;
        }
        blk[i] = iq1bn_encode(t);
      }
    }
  }
  memcpy(out + code_bytes, d, (size_t)n * sizeof(float));
  free(d);
  return ORC_OK;
}

/* IQ1_BN -> int8 T[N,K] and the row scales d[N] (R13). */
int i2s_oracle_iq1bn_unpack(const uint8_t* p, int64_t n, int64_t k, int8_t* t, float* d) {
  if (!p || !t) return ORC_BAD_ARG;
  if (!bn_shape_ok(n, k)) return ORC_BAD_SHAPE;
  int64_t nb = k / BN_BLOCK;
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const uint8_t* blk = p + (r * nb + b) * IQ1BN_BLOCK_BYTES;
      for (int e = 0; e < BN_BLOCK; ++e) {
        int tr = iq1bn_trit(blk[e / 5], e % 5);
        if (tr > 2) return ORC_BAD_CODE;
        t[r * k + b * BN_BLOCK + e] = (int8_t)(tr - 1);
      }
    }
  }
  if (d) memcpy(d, p + n * nb * IQ1BN_BLOCK_BYTES, (size_t)n * sizeof(float));
  return ORC_OK;
}

/* Y[M,N] from ternary T[N,K] with row scales d[N] (R14: R7 with d_n). */
int i2s_oracle_gemm_rows(const int8_t* t, const float* d, int64_t n, int64_t k,
                         const int8_t* xq, const float* xs, int64_t m, float* y, int32_t* acc) {
  if (!t || !d || !xq || !xs) return ORC_BAD_ARG;
  if (n < 1 || k < 1 || m < 1) return ORC_BAD_SHAPE;
  for (int64_t r = 0; r < m; ++r) {
    for (int64_t c = 0; c < n; ++c) {
      int32_t a = 0;
      for (int64_t i = 0; i < k; ++i) {
        int w = t[c * k + i];
        if (w == 1) a += (int32_t)xq[r * k + i];
        else if (w == -1) a -= (int32_t)xq[r * k + i];
      }
      if (acc) acc[r * n + c] = a;
      if (y) {
        float v = (float)a * xs[r];
        y[r * n + c] = v * d[c];
      }
    }
  }
  return ORC_OK;
}
