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
// One CTA per token row (grid-stride).  The row is staged once in shared
// memory as fp32 with 128-bit loads; the RMS mean square is reduced in fp64;
// the FWHT runs its butterfly stages in shared memory in the fixed order
// h = 1, 2, 4, ...; the codes are written with 32-bit stores.  Every fp32
// operation that decides a code is an explicit round-to-nearest intrinsic, so
// no FMA contraction can change a result.
#pragma once

#include "common.cuh"

namespace bitnet {

enum { PRE_NONE = 0, PRE_RMSNORM = 1, PRE_FWHT = 2 };

struct QuantParams {
  const void* X;
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

// Sum of a double and max of a float over the block in one pass (two syncs).
__device__ __forceinline__ void block_sum_max(double& v, float& mx, double* red_d, float* red_f) {
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
  for (int i = 0; i < nw; ++i) {        // fixed order: the same sum in every thread
    w += red_d[i];
    f = fmaxf(f, red_f[i]);
  }
  __syncthreads();
  v = w;
  mx = f;
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

// Prelude value of element k (row[] holds x for NONE / RMSNORM and the
// un-normalised butterfly output for FWHT).
template <int PRE>
__device__ __forceinline__ float prelude_value(float v, int k, float r, const float* gain,
                                               float c) {
  if (PRE == PRE_RMSNORM) {
    float t = __fmul_rn(v, r);
    return gain ? __fmul_rn(t, __ldg(gain + k)) : t;
  } else if (PRE == PRE_FWHT) {
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
    if (PRE == PRE_FWHT) {
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

// Register-resident variant for the NONE and RMSNORM preludes: one CTA per
// token row, NT threads, each holding up to VPT float4 of the row in
// registers.  Every 16-byte load of the row is in flight before the first
// reduction, so the kernel streams at HBM bandwidth; the row is read once.
template <int NT, int VPT, int PRE, bool BF16>
__global__ void __launch_bounds__(NT) quant_act_reg_kernel(QuantParams p) {
  static_assert(PRE == PRE_NONE || PRE == PRE_RMSNORM, "FWHT uses the shared-memory kernel");
  static_assert(!BF16 || VPT % 2 == 0, "bf16 rows load 8 values per 16 bytes");
  __shared__ double red_d[33];
  __shared__ float red_f[33];
  __shared__ int red_i[33];
  const int K = p.K, K4 = p.K / 4;
  const int tid = threadIdx.x;
  for (int m = blockIdx.x; m < p.M; m += gridDim.x) {
    float4 v[VPT];
    if (BF16) {
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const __nv_bfloat16*>(p.X) + (size_t)m * K);
#pragma unroll
      for (int i = 0; i < VPT / 2; ++i) {
        const int idx = tid + i * NT;            // 8-value unit
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (idx < K / 8) u = src[idx];
        v[2 * i] = make_float4(bf16_bits_to_f32(u.x & 0xffffu), bf16_bits_to_f32(u.x >> 16),
                               bf16_bits_to_f32(u.y & 0xffffu), bf16_bits_to_f32(u.y >> 16));
        v[2 * i + 1] = make_float4(bf16_bits_to_f32(u.z & 0xffffu), bf16_bits_to_f32(u.z >> 16),
                                   bf16_bits_to_f32(u.w & 0xffffu), bf16_bits_to_f32(u.w >> 16));
      }
    } else {
      const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.X) +
                                                          (size_t)m * K);
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int idx = tid + i * NT;
        v[i] = idx < K4 ? src[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    // element index of v[i].x: bf16 rows pair float4s inside one 8-value unit
    auto kbase = [&](int i) -> int {
      return BF16 ? 8 * (tid + (i / 2) * NT) + 4 * (i & 1) : 4 * (tid + i * NT);
    };
    float r = 1.0f;
    float amax = 0.0f;
    if (PRE == PRE_RMSNORM) {
      double ss = 0.0;
      float xmax = 0.0f;
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        ss += (double)v[i].x * (double)v[i].x;
        ss += (double)v[i].y * (double)v[i].y;
        ss += (double)v[i].z * (double)v[i].z;
        ss += (double)v[i].w * (double)v[i].w;
        xmax = fmaxf(fmaxf(xmax, fmaxf(fabsf(v[i].x), fabsf(v[i].y))),
                     fmaxf(fabsf(v[i].z), fabsf(v[i].w)));
      }
      if (p.gain == nullptr) {
        // one pass: with r > 0 and no gain, max|fl(x r)| = fl(max|x| r) because
        // rounding is monotone, so the row maximum needs no second reduction
        block_sum_max(ss, xmax, red_d, red_f);
      } else {
        ss = block_sum_f64(ss, red_d);
      }
      const float ms = (float)(ss / (double)K);
      r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.eps)));
      if (p.gain == nullptr) amax = xmax == 0.0f ? 0.0f : __fmul_rn(xmax, r);   // 0 * inf stays 0
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int k = kbase(i);
        if (k < K) {
          float4 g = make_float4(1.f, 1.f, 1.f, 1.f);
          if (p.gain) g = __ldg(reinterpret_cast<const float4*>(p.gain + k));
          v[i].x = __fmul_rn(__fmul_rn(v[i].x, r), g.x);
          v[i].y = __fmul_rn(__fmul_rn(v[i].y, r), g.y);
          v[i].z = __fmul_rn(__fmul_rn(v[i].z, r), g.z);
          v[i].w = __fmul_rn(__fmul_rn(v[i].w, r), g.w);
        }
      }
    }
    if (PRE == PRE_NONE || p.gain != nullptr) {
#pragma unroll
      for (int i = 0; i < VPT; ++i)
        amax = fmaxf(fmaxf(fmaxf(amax, fabsf(v[i].x)), fmaxf(fabsf(v[i].y), fabsf(v[i].z))),
                     fabsf(v[i].w));
      amax = block_max_f32(amax, red_f);
    }
    float s = __fdiv_rn(127.0f, amax);
    const bool zero_row = (amax == 0.0f) || isinf(s);
    if (zero_row) s = 1.0f;
    int rsum = 0;
    uint32_t* dst = reinterpret_cast<uint32_t*>(p.Xq + (size_t)m * K);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int k = kbase(i);
      if (k < K) {
        int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
        if (!zero_row) {
          q0 = quant_code(v[i].x, s);
          q1 = quant_code(v[i].y, s);
          q2 = quant_code(v[i].z, s);
          q3 = quant_code(v[i].w, s);
        }
        rsum += q0 + q1 + q2 + q3;
        dst[k / 4] = (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) |
                     ((uint32_t)(q2 & 0xff) << 16) | ((uint32_t)(q3 & 0xff) << 24);
      }
    }
    if (p.rowsum != nullptr) rsum = block_sum_i32(rsum, red_i);
    if (tid == 0) {
      p.scale[m] = s;
      if (p.rowsum != nullptr) p.rowsum[m] = rsum;
    }
  }
}

}  // namespace bitnet
