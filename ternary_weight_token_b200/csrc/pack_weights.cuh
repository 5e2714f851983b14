// pack_weights.cuh -- absmean ternarisation of a weight matrix and packing of
// the ternary codes four to a byte.
//
// nnterp encyclopedia "bitnet", "The projections quantize their inputs and
// weights": weights are rounded to {-1, 0, 1} * mean|W|; the packed
// checkpoint stores them ternary, four to a byte, with a weight_scale.
// "BitNet b1.58 2B4T", "Model Details": absmean quantisation.
//
// Three launches on the caller's stream:
//   1. absmean_partial: a fixed grid sums |W| in fp64, one partial per CTA in
//      a fixed order (deterministic run to run);
//   2. absmean_final: one CTA adds the partials in a fixed order and writes
//      gamma = fp32(sum / count);
//   3. pack: one thread per 32-bit output word (16 weights), reading gamma
//      from device memory, so the whole chain needs no host synchronisation.
#pragma once

#include "common.cuh"
#include "quant_act.cuh"

namespace bitnet {

constexpr int kPackPartialBlocks = 592;   // 4 x 148 SMs; fixed => deterministic
constexpr int kPackThreads = 256;

template <bool BF16>
__global__ void __launch_bounds__(kPackThreads) absmean_partial_kernel(const void* W,
                                                                       long long count,
                                                                       double* partials) {
  __shared__ double red[33];
  double acc = 0.0;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (BF16) {
    const uint4* v8 = reinterpret_cast<const uint4*>(W);
    const long long nv = count / 8;
    for (long long i = t0; i < nv; i += stride) {
      uint4 v = v8[i];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc += fabs((double)bf16_bits_to_f32(w[j] & 0xffffu));
        acc += fabs((double)bf16_bits_to_f32(w[j] >> 16));
      }
    }
    const uint16_t* s = reinterpret_cast<const uint16_t*>(W);
    for (long long i = nv * 8 + t0; i < count; i += stride)
      acc += fabs((double)bf16_bits_to_f32(s[i]));
  } else {
    const float4* v4 = reinterpret_cast<const float4*>(W);
    const long long nv = count / 4;
    for (long long i = t0; i < nv; i += stride) {
      float4 v = v4[i];
      acc += fabs((double)v.x);
      acc += fabs((double)v.y);
      acc += fabs((double)v.z);
      acc += fabs((double)v.w);
    }
    const float* s = reinterpret_cast<const float*>(W);
    for (long long i = nv * 4 + t0; i < count; i += stride) acc += fabs((double)s[i]);
  }
  acc = block_sum_f64(acc, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = acc;
}

__global__ void __launch_bounds__(kPackThreads) absmean_final_kernel(const double* partials,
                                                                     int nparts,
                                                                     long long count,
                                                                     float* gamma) {
  __shared__ double red[33];
  double acc = 0.0;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) acc += partials[i];
  acc = block_sum_f64(acc, red);
  if (threadIdx.x == 0) *gamma = count > 0 ? (float)(acc / (double)count) : 0.0f;
}

__device__ __forceinline__ uint32_t ternary_code(float w, float g) {
  if (g == 0.0f) return 1u;                         // t = 0
  float r = __fdiv_rn(w, g);                        // IEEE fp32 division
  r = fminf(fmaxf(r, -2.0f), 2.0f);                 // keep rint in range
  float t = rintf(r);                               // half to even
  t = fminf(fmaxf(t, -1.0f), 1.0f);
  return (uint32_t)((int)t + 1);                    // stored code c = t + 1
}

// One thread per 32-bit word of the packed layout: word w of row n holds
// weights k = 16w + 4i + j at byte j, bits 2i (c = t + 1).
template <bool BF16>
__global__ void __launch_bounds__(kPackThreads) pack_kernel(const void* W, int N, int K,
                                                            int ldw, const float* gamma,
                                                            uint8_t* packed) {
  const int words_per_row = ldw / 4;
  const long long total = (long long)N * words_per_row;
  const float g = *gamma;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(idx / words_per_row);
    const int wi = (int)(idx % words_per_row);
    const int k0 = 16 * wi;
    uint32_t word = 0x55555555u;                    // padding: code 1 everywhere
    if (k0 < K) {                                   // K % 16 == 0: a word is all in or all out
      float w[16];
      if (BF16) {
        const uint4* src = reinterpret_cast<const uint4*>(
            reinterpret_cast<const uint16_t*>(W) + (size_t)n * K + k0);
        uint4 a = src[0], b = src[1];
        const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          w[2 * j] = bf16_bits_to_f32(u[j] & 0xffffu);
          w[2 * j + 1] = bf16_bits_to_f32(u[j] >> 16);
        }
      } else {
        const float4* src = reinterpret_cast<const float4*>(
            reinterpret_cast<const float*>(W) + (size_t)n * K + k0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float4 v = src[j];
          w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
        }
      }
      word = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          word |= ternary_code(w[4 * i + j], g) << (8 * j + 2 * i);
    }
    reinterpret_cast<uint32_t*>(packed + (size_t)n * ldw)[wi] = word;
  }
}

// ---------------------------------------------------------------------------
// Canonical exchange layout TW2 <-> the device layout.  Both keep 16 codes in
// each 32-bit word of a row: the device layout holds weight 4i + j of the word
// at bits 8j + 2i (so (word >> 2i) & 0x03030303 gives four byte codes), TW2
// at bits 8i + 2j (byte i = weights 4i .. 4i + 3, low bits first).  The
// conversion transposes that 4 x 4 grid of 2-bit fields and is its own
// inverse.  One thread per word.
__device__ __forceinline__ uint32_t transpose_code_grid(uint32_t w) {
  uint32_t o = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) o |= ((w >> (8 * j + 2 * i)) & 3u) << (8 * i + 2 * j);
  return o;
}

// device layout (rows of ldw bytes) -> TW2 (rows of K / 4 bytes)
__global__ void export_tw2_kernel(const uint32_t* __restrict__ packed, int N, int ldw_words,
                                  int tw2_words, uint32_t* __restrict__ tw2) {
  const int64_t total = (int64_t)N * tw2_words;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = i / tw2_words, w = i - n * tw2_words;
    tw2[i] = transpose_code_grid(packed[n * ldw_words + w]);
  }
}

// TW2 -> device layout; the padded words past K hold code 1 (t = 0)
__global__ void import_tw2_kernel(const uint32_t* __restrict__ tw2, int N, int ldw_words,
                                  int tw2_words, uint32_t* __restrict__ packed) {
  const int64_t total = (int64_t)N * ldw_words;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = i / ldw_words, w = i - n * ldw_words;
    packed[i] = w < tw2_words ? transpose_code_grid(tw2[n * tw2_words + w]) : 0x55555555u;
  }
}

}  // namespace bitnet
