// quant_act.cuh -- per-token absmax int8 activation quantisation with an
// optional fused prelude (RMSNorm or normalised fast Walsh-Hadamard
// transform).
//
// nnterp encyclopedia "bitnet", "The projections quantize their inputs and
// weights": every projection rounds its input per token to 255 levels,
// round(x * 127 / max|x|).  "BitNet b1.58 2B4T", "Model Details": absmax
// quantisation per token.  The RMSNorm prelude is the sub-norm that sits right
// before o_proj / down_proj (nnterp "bitnet", "The block, in order"), and the
// Hadamard prelude is the H-BitLinear input transform ("bitnetv2-model"
// README, "Special Features").
//
// One CTA per token row (grid-stride).  The NONE and RMSNORM preludes keep
// the row in registers (quant_act_reg_kernel: every 16-byte load in flight
// before the first reduction, one exact fp64 FMA per element for the mean
// square, codes rounded by one fp32 add and packed by byte permutes).  The
// FWHT prelude stages the row in shared memory as fp32 and runs its butterfly
// stages there in the fixed order h = 1, 2, 4, ... (quant_act_kernel).  Every
// fp32 operation that decides a code is an explicit round-to-nearest
// intrinsic, so no FMA contraction can change a result.
#pragma once

#include "common.cuh"

namespace bitnet {

// PRE_GLU_RMSNORM: the row is m = relu(g)^2 * u of two fp32 inputs (gate
// X, up X2), as the fused gate/up epilogue forms it, then RMSNorm.
// PRE_SILU_FWHT: the row is silu(x) of the loaded values, then the FWHT (the
// H-BitLinear FFN's hidden activation: the first projection stores its plain
// dequantised output and the second projection's quantiser applies the SiLU
// as it loads it).
enum { PRE_NONE = 0, PRE_RMSNORM = 1, PRE_FWHT = 2, PRE_GLU_RMSNORM = 3, PRE_SILU_FWHT = 4 };

__host__ __device__ constexpr bool is_fwht(int pre) { return pre == PRE_FWHT || pre == PRE_SILU_FWHT; }

struct QuantParams {
  const void* X;
  const float* X2;     // up projection for PRE_GLU_RMSNORM, else unused
  int M, K;
  const float* gain;   // [K] or null (RMSNorm only)
  float eps;           // RMSNorm epsilon
  float fwht_c;        // fp32(1/sqrt(K)) for the FWHT prelude
  int8_t* Xq;
  float* scale;
  int32_t* rowsum;     // may be null
};

// Deterministic block sum of a double: fixed xor-shuffle tree inside each
// warp, then warp 0 adds the per-warp partials in a fixed tree.  Every thread
// receives the result.
__device__ __forceinline__ double block_sum_f64(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    double w = lane < nw ? red[lane] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
    if (lane == 0) red[32] = w;
  }
  __syncthreads();
  double r = red[32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ float block_max_f32(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float w = lane < nw ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, o));
    if (lane == 0) red[32] = w;
  }
  __syncthreads();
  float r = red[32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ int block_sum_i32(int v, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? red[lane] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
    if (lane == 0) red[32] = w;
  }
  __syncthreads();
  int r = red[32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

__device__ __forceinline__ int quant_code(float xh, float s) {
  int q = __float2int_rn(__fmul_rn(xh, s));   // round half to even
  return min(127, max(-128, q));
}

// Codes of four scaled values y = fl(xh * s), packed little-endian.  For
// |y| < 2^22 the fp32 sum 1.5 * 2^23 + y lies in a binade of spacing 1, so its
// round-to-nearest-even is exactly rint(y), and the low byte of its bit
// pattern is rint(y) mod 256.  |y| <= 127 (within rounding) holds for every
// element of a row because s = fl(127 / amax) and |xh| <= amax, so the clamp
// to [-128, 127] of the definition never binds and is not applied.
__device__ __forceinline__ uint32_t pack_codes4(float y0, float y1, float y2, float y3) {
  const float kMagic = 12582912.0f;
  const uint32_t a = __float_as_uint(__fadd_rn(y0, kMagic));
  const uint32_t b = __float_as_uint(__fadd_rn(y1, kMagic));
  const uint32_t c = __float_as_uint(__fadd_rn(y2, kMagic));
  const uint32_t d = __float_as_uint(__fadd_rn(y3, kMagic));
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Prelude value of element k (row[] holds x for NONE / RMSNORM and the
// un-normalised butterfly output for FWHT).
template <int PRE>
__device__ __forceinline__ float prelude_value(float v, int k, float r, const float* gain,
                                               float c) {
  if (PRE == PRE_RMSNORM) {
    float t = __fmul_rn(v, r);
    return gain ? __fmul_rn(t, __ldg(gain + k)) : t;
  } else if (is_fwht(PRE)) {
    return __fmul_rn(v, c);
  }
  return v;
}

template <int PRE, bool BF16>
__global__ void __launch_bounds__(256) quant_act_kernel(QuantParams p) {
  extern __shared__ float4 quant_smem[];
  float* row = reinterpret_cast<float*>(quant_smem);
  __shared__ double red_d[33];
  __shared__ float red_f[33];
  __shared__ int red_i[33];

  const int K = p.K;
  const int tid = threadIdx.x, nt = blockDim.x;
  // launched with programmatic dependent launch: no global access before the
  // preceding grid completed; the next grid may launch only after that (so a
  // GEMM behind this kernel that loads its weights early never overlaps work
  // from before it)
  grid_dependency_wait();
  grid_launch_dependents();
  for (int m = blockIdx.x; m < p.M; m += gridDim.x) {
    // 1. stage the row as fp32; the RMS sum of squares is exact per term in fp64
    double ss = 0.0;
    if (BF16) {
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const __nv_bfloat16*>(p.X) + (size_t)m * K);
      for (int i = tid; i < K / 8; i += nt) {
        uint4 v = src[i];
        float f[8];
        f[0] = bf16_bits_to_f32(v.x & 0xffffu); f[1] = bf16_bits_to_f32(v.x >> 16);
        f[2] = bf16_bits_to_f32(v.y & 0xffffu); f[3] = bf16_bits_to_f32(v.y >> 16);
        f[4] = bf16_bits_to_f32(v.z & 0xffffu); f[5] = bf16_bits_to_f32(v.z >> 16);
        f[6] = bf16_bits_to_f32(v.w & 0xffffu); f[7] = bf16_bits_to_f32(v.w >> 16);
        if (PRE == PRE_SILU_FWHT) {
#pragma unroll
          for (int j = 0; j < 8; ++j) f[j] = silu_f32(f[j]);
        }
        reinterpret_cast<float4*>(row)[2 * i] = make_float4(f[0], f[1], f[2], f[3]);
        reinterpret_cast<float4*>(row)[2 * i + 1] = make_float4(f[4], f[5], f[6], f[7]);
        if (PRE == PRE_RMSNORM) {
#pragma unroll
          for (int j = 0; j < 8; ++j) ss += (double)f[j] * (double)f[j];
        }
      }
    } else {
      const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.X) +
                                                          (size_t)m * K);
      for (int i = tid; i < K / 4; i += nt) {
        float4 v = src[i];
        if (PRE == PRE_SILU_FWHT) {
          v.x = silu_f32(v.x); v.y = silu_f32(v.y); v.z = silu_f32(v.z); v.w = silu_f32(v.w);
        }
        reinterpret_cast<float4*>(row)[i] = v;
        if (PRE == PRE_RMSNORM) {
          ss += (double)v.x * (double)v.x;
          ss += (double)v.y * (double)v.y;
          ss += (double)v.z * (double)v.z;
          ss += (double)v.w * (double)v.w;
        }
      }
    }
    // 2. prelude
    float r = 1.0f;
    if (PRE == PRE_RMSNORM) {
      ss = block_sum_f64(ss, red_d);          // ends with __syncthreads: row is staged
      const float ms = (float)(ss / (double)K);
      r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.eps)));
    } else {
      __syncthreads();
    }
    if (is_fwht(PRE)) {
      for (int h = 1; h < K; h <<= 1) {
        for (int b = tid; b < K / 2; b += nt) {
          const int j = (b / h) * 2 * h + (b % h);
          const float a = row[j], c = row[j + h];
          row[j] = __fadd_rn(a, c);
          row[j + h] = __fsub_rn(a, c);
        }
        __syncthreads();
      }
    }
    // 3. absmax of the prelude output
    float amax = 0.0f;
    for (int g = tid; g < K / 4; g += nt) {
      const float4 v = reinterpret_cast<const float4*>(row)[g];
      const int k = 4 * g;
      amax = fmaxf(amax, fabsf(prelude_value<PRE>(v.x, k + 0, r, p.gain, p.fwht_c)));
      amax = fmaxf(amax, fabsf(prelude_value<PRE>(v.y, k + 1, r, p.gain, p.fwht_c)));
      amax = fmaxf(amax, fabsf(prelude_value<PRE>(v.z, k + 2, r, p.gain, p.fwht_c)));
      amax = fmaxf(amax, fabsf(prelude_value<PRE>(v.w, k + 3, r, p.gain, p.fwht_c)));
    }
    amax = block_max_f32(amax, red_f);
    float s = __fdiv_rn(127.0f, amax);
    const bool zero_row = (amax == 0.0f) || isinf(s);
    if (zero_row) s = 1.0f;
    // 4. codes
    int rsum = 0;
    uint32_t* dst = reinterpret_cast<uint32_t*>(p.Xq + (size_t)m * K);
    for (int g = tid; g < K / 4; g += nt) {
      const float4 v = reinterpret_cast<const float4*>(row)[g];
      const int k = 4 * g;
      int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
      if (!zero_row) {
        q0 = quant_code(prelude_value<PRE>(v.x, k + 0, r, p.gain, p.fwht_c), s);
        q1 = quant_code(prelude_value<PRE>(v.y, k + 1, r, p.gain, p.fwht_c), s);
        q2 = quant_code(prelude_value<PRE>(v.z, k + 2, r, p.gain, p.fwht_c), s);
        q3 = quant_code(prelude_value<PRE>(v.w, k + 3, r, p.gain, p.fwht_c), s);
      }
      rsum += q0 + q1 + q2 + q3;
      dst[g] = (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) |
               ((uint32_t)(q2 & 0xff) << 16) | ((uint32_t)(q3 & 0xff) << 24);
    }
    if (p.rowsum != nullptr) rsum = block_sum_i32(rsum, red_i);
    if (tid == 0) {
      p.scale[m] = s;
      if (p.rowsum != nullptr) p.rowsum[m] = rsum;
    }
    __syncthreads();   // row[] is reused by the next token
  }
}

// ---------------------------------------------------------------------------
// Register-resident rows (NONE and RMSNORM preludes).
//
// Thread t of an NT-thread CTA holds VPT float4 of the row: chunk i is the
// 16-byte unit t + i * NT of an fp32 row, or for a bf16 row, chunks 2j and 2j+1
// are the two halves of the 8-value unit t + j * NT.  Chunks past the end of
// the row hold zeros.  Per element the row costs one exact fp64 FMA of x^2
// (the square of a 24-bit significand is exact in fp64), one |x| max, the
// fp32 products of the definition, one add that rounds, and a quarter of a
// byte permute, dp4a and store each.

template <int NT, int VPT, bool BF16>
__device__ __forceinline__ bool chunk_valid(int i, int K) {
  return BF16 ? (int)threadIdx.x + (i / 2) * NT < K / 8 : (int)threadIdx.x + i * NT < K / 4;
}

template <int NT, int VPT, bool BF16>
__device__ __forceinline__ int chunk_elem(int i) {
  return BF16 ? 8 * ((int)threadIdx.x + (i / 2) * NT) + 4 * (i & 1)
              : 4 * ((int)threadIdx.x + i * NT);
}

// One barrier: warp partials of an fp64 sum and an fp32 max, combined by every
// thread in the same fixed order.  The caller alternates between two partial
// buffers on consecutive rows (and has another barrier per row), so a row's
// partials are never overwritten while a thread still reads them.
__device__ __forceinline__ void block_sum_max_1(double& v, float& mx, double* red_d,
                                                float* red_f) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v += __shfl_xor_sync(0xffffffffu, v, o);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    red_d[warp] = v;
    red_f[warp] = mx;
  }
  __syncthreads();
  double w = 0.0;
  float f = 0.0f;
  for (int i = 0; i < nw; ++i) {
    w += red_d[i];
    f = fmaxf(f, red_f[i]);
  }
  v = w;
  mx = f;
}

__device__ __forceinline__ float block_max_1(float mx, float* red_f) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red_f[warp] = mx;
  __syncthreads();
  float f = 0.0f;
  for (int i = 0; i < nw; ++i) f = fmaxf(f, red_f[i]);
  return f;
}

__device__ __forceinline__ double block_sum_1(double v, double* red_d) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red_d[warp] = v;
  __syncthreads();
  double w = 0.0;
  for (int i = 0; i < nw; ++i) w += red_d[i];
  return w;
}

// Reduction scratch of the register kernels: two alternating buffers of warp
// partials (fp64 sum, fp32 max, fp32 max of a second reduction) and the warp
// partials of the code sum.
struct RowRed {
  double d[2][32];
  float f[2][32];
  float g[2][32];
  int rs[32];
};

// Statistics, scale and codes of row m held in v[]; leaves the warp partials
// of the code sum in red.rs (lane 0 of each warp) for the caller to add up
// after its next barrier.
template <int NT, int VPT, int PRE, bool BF16>
__device__ __forceinline__ void quant_row(const QuantParams& p, int m, float4 (&v)[VPT],
                                          RowRed& red, int par) {
  constexpr bool RMS = PRE == PRE_RMSNORM || PRE == PRE_GLU_RMSNORM;
  const int K = p.K;
  float r = 1.0f, amax = 0.0f;
  if (RMS) {
    double s0 = 0.0, s1 = 0.0;
    float xmax = 0.0f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      s0 = fma((double)v[i].x, (double)v[i].x, s0);
      s1 = fma((double)v[i].y, (double)v[i].y, s1);
      s0 = fma((double)v[i].z, (double)v[i].z, s0);
      s1 = fma((double)v[i].w, (double)v[i].w, s1);
      xmax = fmaxf(xmax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)),
                               fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
    }
    double ss = s0 + s1;
    block_sum_max_1(ss, xmax, red.d[par], red.f[par]);
    const float ms = (float)(ss / (double)K);
    r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.eps)));
    if (p.gain == nullptr) {
      // with r > 0 and no gain, max|fl(x r)| = fl(max|x| r) (rounding is
      // monotone), so the row maximum needs no second reduction; 0 * inf -> 0
      amax = xmax == 0.0f ? 0.0f : __fmul_rn(xmax, r);
    } else {
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        if (chunk_valid<NT, VPT, BF16>(i, K)) {
          const float4 g = __ldg(reinterpret_cast<const float4*>(p.gain + chunk_elem<NT, VPT, BF16>(i)));
          v[i].x = __fmul_rn(__fmul_rn(v[i].x, r), g.x);
          v[i].y = __fmul_rn(__fmul_rn(v[i].y, r), g.y);
          v[i].z = __fmul_rn(__fmul_rn(v[i].z, r), g.z);
          v[i].w = __fmul_rn(__fmul_rn(v[i].w, r), g.w);
          amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)),
                                   fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
        }
      }
      amax = block_max_1(amax, red.g[par]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < VPT; ++i)
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)),
                               fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
    amax = block_max_1(amax, red.f[par]);
  }
  float s = __fdiv_rn(127.0f, amax);
  const bool zero_row = (amax == 0.0f) || isinf(s);
  if (zero_row) s = 1.0f;
  if (threadIdx.x == 0) p.scale[m] = s;
  // the RMS factor is applied here when no gain was (same two roundings)
  const bool fold_r = RMS && p.gain == nullptr;
  int rsum = 0;
  uint8_t* dst = reinterpret_cast<uint8_t*>(p.Xq) + (size_t)m * K;
  auto codes = [&](const float4& x) -> uint32_t {
    if (fold_r)
      return pack_codes4(__fmul_rn(__fmul_rn(x.x, r), s), __fmul_rn(__fmul_rn(x.y, r), s),
                         __fmul_rn(__fmul_rn(x.z, r), s), __fmul_rn(__fmul_rn(x.w, r), s));
    return pack_codes4(__fmul_rn(x.x, s), __fmul_rn(x.y, s), __fmul_rn(x.z, s),
                       __fmul_rn(x.w, s));
  };
  if (BF16) {
#pragma unroll
    for (int j = 0; j < VPT / 2; ++j) {
      if (chunk_valid<NT, VPT, BF16>(2 * j, K)) {
        uint2 w = make_uint2(0u, 0u);
        if (!zero_row) {
          w.x = codes(v[2 * j]);
          w.y = codes(v[2 * j + 1]);
          rsum = __dp4a((int)w.x, 0x01010101, rsum);
          rsum = __dp4a((int)w.y, 0x01010101, rsum);
        }
        *reinterpret_cast<uint2*>(dst + 8 * ((int)threadIdx.x + j * NT)) = w;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      if (chunk_valid<NT, VPT, BF16>(i, K)) {
        uint32_t w = 0u;
        if (!zero_row) {
          w = codes(v[i]);
          rsum = __dp4a((int)w, 0x01010101, rsum);
        }
        reinterpret_cast<uint32_t*>(dst)[(int)threadIdx.x + i * NT] = w;
      }
    }
  }
  rsum = __reduce_add_sync(0xffffffffu, rsum);
  if ((threadIdx.x & 31) == 0) red.rs[threadIdx.x >> 5] = rsum;
}

// Sum of the warp partials of the code sum of row m (thread 0, after a
// barrier that follows their writes).
__device__ __forceinline__ void finish_rowsum(const QuantParams& p, int m, const RowRed& red) {
  if (threadIdx.x == 0 && p.rowsum != nullptr) {
    int t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red.rs[w];
    p.rowsum[m] = t;
  }
}

template <int NT, int VPT, bool BF16>
__device__ __forceinline__ void unpack_row(const uint4 (&u)[BF16 ? VPT / 2 : VPT],
                                           float4 (&v)[VPT]) {
  if (BF16) {
#pragma unroll
    for (int j = 0; j < VPT / 2; ++j) {
      v[2 * j] = make_float4(__uint_as_float(u[j].x << 16), __uint_as_float(u[j].x & 0xffff0000u),
                             __uint_as_float(u[j].y << 16), __uint_as_float(u[j].y & 0xffff0000u));
      v[2 * j + 1] =
          make_float4(__uint_as_float(u[j].z << 16), __uint_as_float(u[j].z & 0xffff0000u),
                      __uint_as_float(u[j].w << 16), __uint_as_float(u[j].w & 0xffff0000u));
    }
  } else {
#pragma unroll
    for (int i = 0; i < VPT; ++i) v[i] = make_float4(__uint_as_float(u[i].x), __uint_as_float(u[i].y),
                                                    __uint_as_float(u[i].z), __uint_as_float(u[i].w));
  }
}

// One CTA per row (grid-stride): every 16-byte load of the row is issued
// before the first reduction.
template <int NT, int VPT, int PRE, bool BF16>
__global__ void __launch_bounds__(NT) quant_act_reg_kernel(QuantParams p) {
  static_assert(PRE == PRE_NONE || PRE == PRE_RMSNORM || PRE == PRE_GLU_RMSNORM,
                "FWHT uses the shared-memory kernel");
  static_assert(PRE != PRE_GLU_RMSNORM || !BF16, "gate/up rows are fp32");
  static_assert(!BF16 || VPT % 2 == 0, "bf16 rows load 8 values per 16 bytes");
  constexpr int NU = BF16 ? VPT / 2 : VPT;
  __shared__ RowRed red;
  const int K = p.K;
  const int units = BF16 ? K / 8 : K / 4;
  const int row_bytes = K * (BF16 ? 2 : 4);
  // launched with programmatic dependent launch: no global access before the
  // preceding grid completed; the next grid may launch only after that (so a
  // GEMM behind this kernel that loads its weights early never overlaps work
  // from before it)
  grid_dependency_wait();
  grid_launch_dependents();
  int par = 0;
  for (int m = blockIdx.x; m < p.M; m += gridDim.x, par ^= 1) {
    const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(p.X) +
                                                      (size_t)m * row_bytes);
    uint4 u[NU];
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const int idx = (int)threadIdx.x + j * NT;
      u[j] = idx < units ? ld_stream_v4(src + idx) : make_uint4(0u, 0u, 0u, 0u);
    }
    float4 v[VPT];
    unpack_row<NT, VPT, BF16>(u, v);
    if (PRE == PRE_GLU_RMSNORM) {
      // m = relu(g)^2 * u, fp32 products in the epilogue's order
      const float4* up = reinterpret_cast<const float4*>(p.X2 + (size_t)m * K);
      auto glu = [](float g, float x) { return __fmul_rn(g > 0.0f ? __fmul_rn(g, g) : 0.0f, x); };
      uint4 w[VPT];
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int idx = (int)threadIdx.x + i * NT;
        w[i] = idx < units ? ld_stream_v4(up + idx) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < VPT; ++i)
        v[i] = make_float4(glu(v[i].x, __uint_as_float(w[i].x)), glu(v[i].y, __uint_as_float(w[i].y)),
                           glu(v[i].z, __uint_as_float(w[i].z)), glu(v[i].w, __uint_as_float(w[i].w)));
    }
    quant_row<NT, VPT, PRE, BF16>(p, m, v, red, par);
    __syncthreads();
    finish_rowsum(p, m, red);
  }
}

// ---------------------------------------------------------------------------
// FWHT prelude with the row in registers (K = 2^n, VEC * 32 * WPR <= K <=
// 2048), WPR warps per token row (1, 2 or 4; a 128-thread CTA takes 4 / WPR
// rows at a time).  Warp w of a row holds elements k = KW w + 32 VEC j +
// VEC l + e (KW = K / WPR, lane l, vector j, element e of a 16-byte vector).
// The butterfly stages run in the fixed order h = 1, 2, 4, ...: h < VEC
// inside a vector, VEC <= h < 32 VEC between lanes (shuffle with lane ^
// (h / VEC); the lower partner keeps a + b, the upper a - b, the same fp32
// operations as the staged kernel), 32 VEC <= h < KW between a lane's own
// vectors, and h >= KW between the row's warps through shared memory (each
// thread reads the WPR values of its position and runs those stages in the
// same order).  Several warps per row keep more rows in flight and shorten
// each warp's chain of dependent instructions.
template <int K, bool BF16, bool SILU = false, int WPR = 1>
__global__ void __launch_bounds__(128) quant_fwht_warp_kernel(QuantParams p) {
  constexpr int VEC = BF16 ? 8 : 4;
  constexpr int KW = K / WPR;
  constexpr int J = KW / (32 * VEC);
  constexpr int RPC = 4 / WPR;                      // rows per CTA at a time
  static_assert(WPR == 1 || WPR == 2 || WPR == 4, "warps per row");
  static_assert(J >= 1 && J * 32 * VEC * WPR == K, "row width");
  __shared__ float xw[WPR > 1 ? 4 * KW : 1];        // [warp][KW] for the cross-warp stages
  __shared__ float red_f[4];
  __shared__ int red_i[4];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rg = warp / WPR, wr = warp - rg * WPR;  // row slot of the CTA, warp within the row
  // launched with programmatic dependent launch: no global access before the
  // preceding grid completed; the next grid may launch only after that (so a
  // GEMM behind this kernel that loads its weights early never overlaps work
  // from before it)
  grid_dependency_wait();
  grid_launch_dependents();
  for (int m0 = blockIdx.x * RPC; m0 < p.M; m0 += gridDim.x * RPC) {   // same trip count CTA-wide
    const int m = m0 + rg;
    const bool row = m < p.M;
    const size_t rbase = (size_t)(row ? m : 0) * K + (size_t)wr * KW;
    float v[J][VEC];
    if (BF16) {
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint16_t*>(p.X) + rbase) + lane;
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const uint4 u = row ? ld_stream_v4(src + 32 * j) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[j][2 * e] = __uint_as_float(w4[e] << 16);
          v[j][2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
        }
      }
    } else {
      const float4* src = reinterpret_cast<const float4*>(
          reinterpret_cast<const float*>(p.X) + rbase) + lane;
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const uint4 u = row ? ld_stream_v4(src + 32 * j) : make_uint4(0u, 0u, 0u, 0u);
        v[j][0] = __uint_as_float(u.x); v[j][1] = __uint_as_float(u.y);
        v[j][2] = __uint_as_float(u.z); v[j][3] = __uint_as_float(u.w);
      }
    }
    if (SILU) {                    // PRE_SILU_FWHT: the row is silu of the loaded values
#pragma unroll
      for (int j = 0; j < J; ++j)
#pragma unroll
        for (int e = 0; e < VEC; ++e) v[j][e] = silu_f32(v[j][e]);
    }
    // h < VEC: inside each vector
#pragma unroll
    for (int h = 1; h < VEC; h <<= 1)
#pragma unroll
      for (int j = 0; j < J; ++j)
#pragma unroll
        for (int e = 0; e < VEC; ++e)
          if ((e & h) == 0) {
            const float a = v[j][e], b = v[j][e + h];
            v[j][e] = __fadd_rn(a, b);
            v[j][e + h] = __fsub_rn(a, b);
          }
    // VEC <= h < 32 VEC: between lanes
#pragma unroll
    for (int lb = 1; lb < 32; lb <<= 1) {
      const bool upper = (lane & lb) != 0;
#pragma unroll
      for (int j = 0; j < J; ++j)
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float mine = v[j][e];
          const float other = __shfl_xor_sync(0xffffffffu, mine, lb);
          v[j][e] = upper ? __fsub_rn(other, mine) : __fadd_rn(mine, other);
        }
    }
    // 32 VEC <= h < KW: between this lane's vectors
#pragma unroll
    for (int hj = 1; hj < J; hj <<= 1)
#pragma unroll
      for (int j = 0; j < J; ++j)
        if ((j & hj) == 0)
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            const float a = v[j][e], b = v[j + hj][e];
            v[j][e] = __fadd_rn(a, b);
            v[j + hj][e] = __fsub_rn(a, b);
          }
    // h >= KW: between the row's warps
    if constexpr (WPR > 1) {
#pragma unroll
      for (int j = 0; j < J; ++j)
#pragma unroll
        for (int e = 0; e < VEC; ++e) xw[warp * KW + 32 * VEC * j + VEC * lane + e] = v[j][e];
      __syncthreads();
#pragma unroll
      for (int j = 0; j < J; ++j)
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          float t[WPR];
#pragma unroll
          for (int w = 0; w < WPR; ++w) t[w] = xw[(rg * WPR + w) * KW + 32 * VEC * j + VEC * lane + e];
#pragma unroll
          for (int hb = 1; hb < WPR; hb <<= 1)
#pragma unroll
            for (int w = 0; w < WPR; ++w)
              if ((w & hb) == 0) {
                const float a = t[w], b = t[w + hb];
                t[w] = __fadd_rn(a, b);
                t[w + hb] = __fsub_rn(a, b);
              }
          v[j][e] = t[wr];
        }
    }
    // normalisation, absmax, codes
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < J; ++j)
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        v[j][e] = __fmul_rn(v[j][e], p.fwht_c);
        amax = fmaxf(amax, fabsf(v[j][e]));
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if constexpr (WPR > 1) {
      if (lane == 0) red_f[warp] = amax;
      __syncthreads();
#pragma unroll
      for (int w = 0; w < WPR; ++w) amax = fmaxf(amax, red_f[rg * WPR + w]);
    }
    float s = __fdiv_rn(127.0f, amax);
    const bool zero_row = (amax == 0.0f) || isinf(s);
    if (zero_row) s = 1.0f;
    int rsum = 0;
    uint32_t* dst = reinterpret_cast<uint32_t*>(p.Xq + rbase);
#pragma unroll
    for (int j = 0; j < J; ++j)
#pragma unroll
      for (int e = 0; e < VEC; e += 4) {
        uint32_t w = 0u;
        if (!zero_row) {
          w = pack_codes4(__fmul_rn(v[j][e], s), __fmul_rn(v[j][e + 1], s),
                          __fmul_rn(v[j][e + 2], s), __fmul_rn(v[j][e + 3], s));
          rsum = __dp4a((int)w, 0x01010101, rsum);
        }
        if (row) dst[(VEC * lane + 32 * VEC * j + e) / 4] = w;
      }
    rsum = __reduce_add_sync(0xffffffffu, rsum);
    if constexpr (WPR > 1) {
      if (lane == 0) red_i[warp] = rsum;
      __syncthreads();
      if (row && wr == 0 && lane == 0) {
        int t = 0;
#pragma unroll
        for (int w = 0; w < WPR; ++w) t += red_i[rg * WPR + w];
        p.scale[m] = s;
        if (p.rowsum != nullptr) p.rowsum[m] = t;
      }
      __syncthreads();             // xw / red_* are rewritten by the next rows
    } else if (row && lane == 0) {
      p.scale[m] = s;
      if (p.rowsum != nullptr) p.rowsum[m] = rsum;
    }
  }
}

}  // namespace bitnet
