// pack_weights.cuh -- absmean ternarisation of a weight matrix and packing of
// the ternary codes four to a byte.
//
// nnterp encyclopedia "bitnet", "The projections quantize their inputs and
// weights": weights are rounded to {-1, 0, 1} * mean|W|; the packed
// checkpoint stores them ternary, four to a byte, with a weight_scale.
// "BitNet b1.58 2B4T", "Model Details": absmean quantisation.
//
// One cooperative launch (pack_fused_kernel, below) when the device can hold
// its grid at once; otherwise three launches on the caller's stream (with
// programmatic dependent launch: each waits for its predecessor before
// touching global memory):
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
  grid_launch_dependents();       // launched with programmatic dependent launch:
  grid_dependency_wait();         // no global access before the preceding grid completed
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (BF16) {
    // four independent 16-byte loads in flight per thread, four partial sums
    // added in a fixed order
    const uint4* v8 = reinterpret_cast<const uint4*>(W);
    const long long nv = count / 8;
    double a4[4] = {0.0, 0.0, 0.0, 0.0};
    long long i = t0;
    for (; i + 3 * stride < nv; i += 4 * stride) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = ld_stream_v4(v8 + i + u * stride);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          a4[u] += fabs((double)bf16_bits_to_f32(w[j] & 0xffffu));
          a4[u] += fabs((double)bf16_bits_to_f32(w[j] >> 16));
        }
      }
    }
    for (; i < nv; i += stride) {
      uint4 v = v8[i];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        a4[0] += fabs((double)bf16_bits_to_f32(w[j] & 0xffffu));
        a4[0] += fabs((double)bf16_bits_to_f32(w[j] >> 16));
      }
    }
    acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
    const uint16_t* s = reinterpret_cast<const uint16_t*>(W);
    for (long long i = nv * 8 + t0; i < count; i += stride)
      acc += fabs((double)bf16_bits_to_f32(s[i]));
  } else {
    const float4* v4 = reinterpret_cast<const float4*>(W);
    const long long nv = count / 4;
    double a4[4] = {0.0, 0.0, 0.0, 0.0};
    long long i = t0;
    for (; i + 3 * stride < nv; i += 4 * stride) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = ld_stream_v4(v4 + i + u * stride);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a4[u] += fabs((double)__uint_as_float(v[u].x));
        a4[u] += fabs((double)__uint_as_float(v[u].y));
        a4[u] += fabs((double)__uint_as_float(v[u].z));
        a4[u] += fabs((double)__uint_as_float(v[u].w));
      }
    }
    for (; i < nv; i += stride) {
      float4 v = v4[i];
      a4[0] += fabs((double)v.x);
      a4[0] += fabs((double)v.y);
      a4[0] += fabs((double)v.z);
      a4[0] += fabs((double)v.w);
    }
    acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
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
  grid_launch_dependents();
  grid_dependency_wait();
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) acc += partials[i];
  acc = block_sum_f64(acc, red);
  if (threadIdx.x == 0) *gamma = count > 0 ? (float)(acc / (double)count) : 0.0f;
}

// t = clamp(rint(fl(w / g)), -1, 1) without the division.  t != 0 exactly
// when |fl(w / g)| > 1/2; rounding is monotone and the tie 1/2 + 2^-25 rounds
// to the even 1/2, so that holds exactly when |w| > g (1/2 + 2^-25) = T.  T
// is exact in fp64 (a 24-bit significand times a 26-bit one), and for an
// fp32 |w|, |w| > T exactly when |w| > T rounded down to fp32 (thr).  g = 0
// gives t = 0 for every weight.
__device__ __forceinline__ float ternary_threshold(float g) {
  return __double2float_rd((double)g * (0.5 + 0x1p-25));
}

__device__ __forceinline__ uint32_t ternary_code(float w, float g, float thr) {
  if (g == 0.0f || !(fabsf(w) > thr)) return 1u;   // t = 0
  return w > 0.0f ? 2u : 0u;                        // stored code c = t + 1
}

// One thread per 32-bit word of the packed layout: word w of row n holds
// weights k = 16w + 4i + j at byte j, bits 2i (c = t + 1).
template <bool BF16>
__global__ void __launch_bounds__(kPackThreads) pack_kernel(const void* W, int N, int K,
                                                            int ldw, const float* gamma,
                                                            uint8_t* packed) {
  const int words_per_row = ldw / 4;
  const long long total = (long long)N * words_per_row;
  grid_launch_dependents();
  grid_dependency_wait();
  const float g = *gamma;
  const float thr = ternary_threshold(g);
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
        uint4 a = ld_stream_v4(src), b = ld_stream_v4(src + 1);
        const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          w[2 * j] = bf16_bits_to_f32(u[j] & 0xffffu);
          w[2 * j + 1] = bf16_bits_to_f32(u[j] >> 16);
        }
      } else {
        const float4* src = reinterpret_cast<const float4*>(
            reinterpret_cast<const float*>(W) + (size_t)n * K + k0);
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = ld_stream_v4(src + j);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          w[4 * j] = __uint_as_float(v[j].x); w[4 * j + 1] = __uint_as_float(v[j].y);
          w[4 * j + 2] = __uint_as_float(v[j].z); w[4 * j + 3] = __uint_as_float(v[j].w);
        }
      }
      word = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          word |= ternary_code(w[4 * i + j], g, thr) << (8 * j + 2 * i);
    }
    reinterpret_cast<uint32_t*>(packed + (size_t)n * ldw)[wi] = word;
  }
}

// ---------------------------------------------------------------------------
// Both passes in one cooperative launch (every CTA resident): each CTA adds
// |W| over its grid-stride share in fp64 (the same loop as
// absmean_partial_kernel, so the per-CTA order is fixed), publishes its
// partial and the launch's epoch, waits (bounded) for every CTA's epoch, then
// adds all partials in a fixed order -- the same gamma in every CTA, written
// once by CTA 0 -- and packs its share of the codes.  The second read of W
// mostly hits L2: the pass that read it just finished and the matrix is
// smaller than L2.
constexpr int kPackFusedThreads = 512;
constexpr int kPackMaxGrid = 1024;        // partial / flag slots in the workspace
constexpr int kPackWords = 4;             // output words per thread per batch (pass 2)

template <bool BF16>
__global__ void __launch_bounds__(kPackFusedThreads) pack_fused_kernel(
    const void* W, int N, int K, int ldw, long long count, double* partials,
    unsigned long long* flags, unsigned long long epoch, float* gamma_out, uint8_t* packed) {
  __shared__ double red[33];
  __shared__ int xok;
  __shared__ float s_gamma;
  // pass 1: this CTA's partial sum of |W|
  double acc = 0.0;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (BF16) {
    const uint4* v8 = reinterpret_cast<const uint4*>(W);
    const long long nv = count / 8;
    double a4[4] = {0.0, 0.0, 0.0, 0.0};
    long long i = t0;
    for (; i + 3 * stride < nv; i += 4 * stride) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldcg(v8 + i + u * stride);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          a4[u] += fabs((double)bf16_bits_to_f32(w[j] & 0xffffu));
          a4[u] += fabs((double)bf16_bits_to_f32(w[j] >> 16));
        }
      }
    }
    for (; i < nv; i += stride) {
      const uint4 v = __ldcg(v8 + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        a4[0] += fabs((double)bf16_bits_to_f32(w[j] & 0xffffu));
        a4[0] += fabs((double)bf16_bits_to_f32(w[j] >> 16));
      }
    }
    acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
    const uint16_t* sv = reinterpret_cast<const uint16_t*>(W);
    for (long long j = nv * 8 + t0; j < count; j += stride) acc += fabs((double)bf16_bits_to_f32(sv[j]));
  } else {
    const uint4* v4 = reinterpret_cast<const uint4*>(W);
    const long long nv = count / 4;
    double a4[4] = {0.0, 0.0, 0.0, 0.0};
    long long i = t0;
    for (; i + 3 * stride < nv; i += 4 * stride) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldcg(v4 + i + u * stride);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a4[u] += fabs((double)__uint_as_float(v[u].x));
        a4[u] += fabs((double)__uint_as_float(v[u].y));
        a4[u] += fabs((double)__uint_as_float(v[u].z));
        a4[u] += fabs((double)__uint_as_float(v[u].w));
      }
    }
    for (; i < nv; i += stride) {
      const uint4 v = __ldcg(v4 + i);
      a4[0] += fabs((double)__uint_as_float(v.x));
      a4[0] += fabs((double)__uint_as_float(v.y));
      a4[0] += fabs((double)__uint_as_float(v.z));
      a4[0] += fabs((double)__uint_as_float(v.w));
    }
    acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
    const float* sv = reinterpret_cast<const float*>(W);
    for (long long j = nv * 4 + t0; j < count; j += stride) acc += fabs((double)sv[j]);
  }
  acc = block_sum_f64(acc, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = acc;
  // exchange, then gamma from every partial in a fixed order (warp 0: lane l
  // adds partials l, l + 32, ... in turn, then a fixed xor tree)
  const bool ok = grid_exchange(flags, epoch, &xok);
  if (threadIdx.x < 32) {
    // every partial of a lane loaded before any is added (one L2 round trip)
    double pv[kPackMaxGrid / 32];
#pragma unroll
    for (int j = 0; j < kPackMaxGrid / 32; ++j) {
      const int i = (int)threadIdx.x + 32 * j;
      pv[j] = i < (int)gridDim.x ? __ldcg(partials + i) : 0.0;
    }
    double v = 0.0;
#pragma unroll
    for (int j = 0; j < kPackMaxGrid / 32; ++j) v += pv[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) {
      const float g = count > 0 ? (float)(v / (double)count) : 0.0f;
      s_gamma = g;
      if (blockIdx.x == 0 && ok) *gamma_out = g;
    }
  }
  __syncthreads();
  if (!ok) return;
  // pass 2: codes, one thread per 32-bit word of the packed layout; each
  // thread takes kPackWords words of the grid-stride sequence at a time, all
  // their loads (from L2: pass 1 just read them) issued before any is used
  const float g = s_gamma;
  const float thr = ternary_threshold(g);
  const int words_per_row = ldw / 4;
  constexpr int VPW = BF16 ? 2 : 4;               // 16-byte loads per word
  // word index t0 + j * stride as (row, word) without a division per word:
  // one division here, then steps of (stride / wpr, stride % wpr) with a carry
  const long long st_rows = stride / words_per_row;
  const int st_words = (int)(stride - st_rows * words_per_row);
  long long cur_n = t0 / words_per_row;
  int cur_w = (int)(t0 - cur_n * words_per_row);
  while (cur_n < N) {
    uint4 raw[kPackWords][VPW];
    int rown[kPackWords], wordi[kPackWords];
#pragma unroll
    for (int u = 0; u < kPackWords; ++u) {
      rown[u] = -1;
      if (cur_n < N) {
        const int n = (int)cur_n;
        const int wi = cur_w;
        rown[u] = n;
        wordi[u] = wi;
        cur_n += st_rows;
        cur_w += st_words;
        if (cur_w >= words_per_row) {
          cur_w -= words_per_row;
          ++cur_n;
        }
        if (16 * wi < K) {
          const uint4* src = reinterpret_cast<const uint4*>(
              reinterpret_cast<const uint8_t*>(W) + ((size_t)n * K + 16 * (size_t)wi) * (BF16 ? 2 : 4));
#pragma unroll
          for (int j = 0; j < VPW; ++j) raw[u][j] = ld_stream_v4(src + j);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPackWords; ++u) {
      if (rown[u] < 0) continue;
      uint32_t word = 0x55555555u;                  // padding: code 1 everywhere
      if (16 * wordi[u] < K) {
        float w[16];
        if (BF16) {
          const uint32_t v[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                                 raw[u][1].x, raw[u][1].y, raw[u][1].z, raw[u][1].w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            w[2 * j] = bf16_bits_to_f32(v[j] & 0xffffu);
            w[2 * j + 1] = bf16_bits_to_f32(v[j] >> 16);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            w[4 * j] = __uint_as_float(raw[u][j].x); w[4 * j + 1] = __uint_as_float(raw[u][j].y);
            w[4 * j + 2] = __uint_as_float(raw[u][j].z); w[4 * j + 3] = __uint_as_float(raw[u][j].w);
          }
        }
        word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            word |= ternary_code(w[4 * i + j], g, thr) << (8 * j + 2 * i);
      }
      reinterpret_cast<uint32_t*>(packed + (size_t)rown[u] * ldw)[wordi[u]] = word;
    }
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
