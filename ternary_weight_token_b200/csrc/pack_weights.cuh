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

// The stored code c = t + 1 is then 1 when g is 0 or |w| <= thr, else 2 for
// w > 0 and 0 for w < 0.  The forms below give the codes of 16 weights at
// once, as one word of the packed layout, when gamma is finite and positive (then every weight is finite: an infinite
// or NaN weight makes the mean so).  For non-negative floats |w| > thr exactly
// when the magnitude bits of w exceed the bits of thr, and adding
// (field maximum - thr bits) to the magnitude sets the field's top bit exactly
// then, with no carry out of the field: one add gives a weight's nonzero flag,
// its sign bit its sign.  Byte permutes gather the flags of weights
// 4i .. 4i + 3 into bit 7 of bytes 0 .. 3, shifts move them to bit 2i + 1.
// With a = nonzero and b = sign there, the code c = t + 1 is 2 (a, not b),
// 0 (a and b) or 1 (not a): bit 2i + 1 = a & ~b, bit 2i = ~a.
//
// bf16: word p of w holds weights 2p (low half) and 2p + 1 (high half), and
// d2 = 0x7fff - (thr bits >> 16) in both halves.  A bf16 magnitude m (the
// fp32 bits m << 16) exceeds thr exactly when m > (thr bits >> 16), and
// m + d2 <= 0x7f7f + 0x7fff stays inside its 16-bit half.
// bf16: the 8 weights of x (four 32-bit words, weight 2p in the low half of
// word p) are weights 4i .. 4i + 7 of a packed word (i = 0 or 2); their
// nonzero and sign flags go to bits 2i + 1 and 2i + 3 of each byte of a, b.
// d2 = 0x7fff - (thr bits >> 16) in both halves: a bf16 magnitude m (the fp32
// bits m << 16) exceeds thr exactly when m > (thr bits >> 16), and
// m + d2 <= 0x7f7f + 0x7fff stays inside its 16-bit half.
__device__ __forceinline__ void ternary_flags_bf16(const uint4& x, int i, uint32_t d2,
                                                   uint32_t& a, uint32_t& b) {
  // byte j of each permute: the top byte of weight 4i + j (4i + 4 + j)
  const uint32_t nz0 = __byte_perm((x.x & 0x7fff7fffu) + d2, (x.y & 0x7fff7fffu) + d2, 0x7531);
  const uint32_t nz1 = __byte_perm((x.z & 0x7fff7fffu) + d2, (x.w & 0x7fff7fffu) + d2, 0x7531);
  const uint32_t sg0 = __byte_perm(x.x, x.y, 0x7531), sg1 = __byte_perm(x.z, x.w, 0x7531);
  const uint32_t m0 = 0x02020202u << (2 * i), m1 = m0 << 2;
  a |= ((nz0 >> (6 - 2 * i)) & m0) | ((nz1 >> (4 - 2 * i)) & m1);
  b |= ((sg0 >> (6 - 2 * i)) & m0) | ((sg1 >> (4 - 2 * i)) & m1);
}

// fp32: x holds weights 4i .. 4i + 3 of a packed word; d = 0x7fffffff - thr
// bits (the sum stays below 2^32 for finite magnitudes).
__device__ __forceinline__ void ternary_flags_f32(const uint4& x, int i, uint32_t d, uint32_t& a,
                                                  uint32_t& b) {
  const uint32_t n01 = __byte_perm((x.x & 0x7fffffffu) + d, (x.y & 0x7fffffffu) + d, 0x0073);
  const uint32_t n23 = __byte_perm((x.z & 0x7fffffffu) + d, (x.w & 0x7fffffffu) + d, 0x0073);
  const uint32_t nz = __byte_perm(n01, n23, 0x5410);   // byte j: top byte of weight 4i + j
  const uint32_t sg =
      __byte_perm(__byte_perm(x.x, x.y, 0x0073), __byte_perm(x.z, x.w, 0x0073), 0x5410);
  const uint32_t m = 0x02020202u << (2 * i);
  a |= (nz >> (6 - 2 * i)) & m;
  b |= (sg >> (6 - 2 * i)) & m;
}

// the packed word from the flags: bit 2i + 1 = a & ~b, bit 2i = ~a
__device__ __forceinline__ uint32_t ternary_word_from_flags(uint32_t a, uint32_t b) {
  return (a & ~b) | (~(a >> 1) & 0x55555555u);
}

// One packed word from its 16 weights as 16-byte units in order.
template <bool BF16>
__device__ __forceinline__ uint32_t ternary_word(const uint4* x, uint32_t dcode) {
  uint32_t a = 0u, b = 0u;
  if (BF16) {
    ternary_flags_bf16(x[0], 0, dcode, a, b);
    ternary_flags_bf16(x[1], 2, dcode, a, b);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) ternary_flags_f32(x[i], i, dcode, a, b);
  }
  return ternary_word_from_flags(a, b);
}

// dcode of the forms above for threshold bits thr_bits
template <bool BF16>
__device__ __forceinline__ uint32_t ternary_dcode(uint32_t thr_bits) {
  return BF16 ? (0x7fffu - (thr_bits >> 16)) * 0x00010001u : 0x7fffffffu - thr_bits;
}

// gamma for which the word forms above apply (finite, positive)
__device__ __forceinline__ bool gamma_codes_live(float g) { return g > 0.0f && g <= 3.402823466e38f; }

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
  const bool live = gamma_codes_live(g);
  const uint32_t thr_bits = __float_as_uint(ternary_threshold(g));
  const uint32_t dcode = ternary_dcode<BF16>(thr_bits);
  constexpr int UPW = BF16 ? 2 : 4;                 // 16-byte units per word
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(idx / words_per_row);
    const int wi = (int)(idx % words_per_row);
    const int k0 = 16 * wi;
    uint32_t word = 0x55555555u;                    // padding, or gamma 0: code 1 everywhere
    if (k0 < K && live) {                           // K % 16 == 0: a word is all in or all out
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint8_t*>(W) + ((size_t)n * K + k0) * (BF16 ? 2 : 4));
      uint4 x[UPW];
#pragma unroll
      for (int j = 0; j < UPW; ++j) x[j] = ld_stream_v4(src + j);
      word = ternary_word<BF16>(x, dcode);
    }
    reinterpret_cast<uint32_t*>(packed + (size_t)n * ldw)[wi] = word;
  }
}

// ---------------------------------------------------------------------------
// Both passes in one cooperative launch (every CTA resident).  CTA c owns a
// contiguous share of the packed words, whose weights are one contiguous run
// of W; the first smem_bytes of that run are bulk-copied into shared memory
// at the start and stay there for the second pass (the rest is read from
// global memory twice, the second time mostly from L2).
//   pass 1: the CTA adds |W| over its run in fp64 in a fixed order and
//           publishes the partial sum, split over two words tagged with the
//           launch's epoch (64-bit stores are single-copy atomic, so a word
//           that shows this launch's tag holds this launch's half);
//   CTA 0 waits (bounded) until every CTA's two words carry the tag, adds the
//           partials in a fixed order and publishes gamma in two tagged words;
//   pass 2: every CTA waits (bounded) for gamma and writes its words' codes.
// Workspace: 2 kPackMaxGrid partial words and the two gamma words, none of
// which needs initialising (epochs are never reused).
constexpr int kPackFusedThreads = 512;
constexpr int kPackMaxGrid = 1024;        // CTAs of the launch at most
constexpr int kPackMaxStage = 128 * 1024;  // bytes of weights a CTA keeps in shared memory, at most
constexpr int kPackWordsBf16 = 2;         // output words per thread per batch (pass 2)
constexpr int kPackWordsF32 = 2;

template <bool BF16>
__device__ __forceinline__ void add_abs_unit(double& acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (BF16) {
      acc += fabs((double)bf16_bits_to_f32(w[j] & 0xffffu));
      acc += fabs((double)bf16_bits_to_f32(w[j] >> 16));
    } else {
      acc += fabs((double)__uint_as_float(w[j]));
    }
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kPackFusedThreads, 2) pack_fused_kernel(
    const void* W, int N, int K, int ldw, long long count, unsigned long long* xw,
    unsigned long long epoch, int smem_bytes, float* gamma_out, uint8_t* packed) {
  extern __shared__ __align__(128) uint8_t pk_smem[];
  __shared__ double red[33];
  __shared__ int xok;
  __shared__ float s_gamma;
  constexpr int WB = BF16 ? 32 : 64;              // bytes of the 16 weights of one packed word
  constexpr int UPW = WB / 16;                    // 16-byte units per word
  constexpr int kPackWords = BF16 ? kPackWordsBf16 : kPackWordsF32;
  const int tid = threadIdx.x, lane = tid & 31;
  const int wpr = ldw / 4, kw = K / 16;           // words per packed row; of them with weights
  const long long total = (long long)N * wpr;
  const long long q0 = total * blockIdx.x / gridDim.x;
  const long long q1 = total * (blockIdx.x + 1) / gridDim.x;
  // weights (in words of 16) before packed word q: whole rows, then the
  // row's words that hold weights (padding words hold none)
  auto src_of = [&](long long q) {
    const long long n = q / wpr;
    const int wi = (int)(q - n * wpr);
    return n * kw + (wi < kw ? wi : kw);
  };
  const long long s0 = src_of(q0), nsrc = src_of(q1) - s0;
  const int ns = (int)(nsrc < smem_bytes / WB ? nsrc : smem_bytes / WB);   // words staged
  const uint8_t* gsrc = reinterpret_cast<const uint8_t*>(W) + s0 * WB;
  // pass 1: thread t takes the 16-byte units t, t + 512, ... of the run in
  // groups of 4, unit 4 j + k of its sequence into fp64 sum k (a fixed
  // order); the next group's loads are issued before the current group is
  // added (the conversions to fp64 run at a fraction of the load rate, so
  // they must overlap the loads), and units of the staged words are also
  // stored to shared memory for pass 2
  const uint4* g16 = reinterpret_cast<const uint4*>(gsrc);
  const int nunits = (int)(nsrc * UPW), sunits = ns * UPW;
  uint4* s16 = reinterpret_cast<uint4*>(pk_smem);
  double a4[4] = {0.0, 0.0, 0.0, 0.0};
  uint4 cur[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int u = tid + k * kPackFusedThreads;
    cur[k] = u < nunits ? __ldcg(g16 + u) : make_uint4(0u, 0u, 0u, 0u);   // zeros add nothing
  }
  for (int u0 = tid; u0 < nunits; u0 += 4 * kPackFusedThreads) {
    uint4 nxt[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int u = u0 + (4 + k) * kPackFusedThreads;
      nxt[k] = u < nunits ? __ldcg(g16 + u) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int u = u0 + k * kPackFusedThreads;
      if (u < sunits) s16[u] = cur[k];
      add_abs_unit<BF16>(a4[k], cur[k]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) cur[k] = nxt[k];
  }
  double acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
  acc = block_sum_f64(acc, red);
  const int G = (int)gridDim.x;
  const unsigned long long tag = (epoch & 0xffffffffull) << 32, hi_mask = ~0xffffffffull;
  unsigned long long* gwords = xw + 2 * kPackMaxGrid;
  if (tid == 0) {
    const unsigned long long pb = (unsigned long long)__double_as_longlong(acc);
    st_relaxed_u64(xw + 2 * blockIdx.x, tag | (pb & 0xffffffffull));
    st_relaxed_u64(xw + 2 * blockIdx.x + 1, tag | (pb >> 32));
  }
  static_assert(kPackMaxGrid <= 2 * kPackFusedThreads, "two partials per thread of CTA 0");
  if (blockIdx.x == 0) {
    // thread t reads the words of CTAs t and t + 512 (one L2 round trip per
    // poll for the whole CTA); the decisions to stop are CTA-wide
    const int t2 = tid + kPackFusedThreads;
    const unsigned long long tw0 = global_timer_ns();
    bool done = false;
    double v = 0.0;
    for (uint32_t it = 0;; ++it) {
      unsigned long long a0 = tag, a1 = tag, b0 = tag, b1 = tag;
      if (tid < G) {
        a0 = ld_relaxed_u64(xw + 2 * tid);
        a1 = ld_relaxed_u64(xw + 2 * tid + 1);
      }
      if (t2 < G) {
        b0 = ld_relaxed_u64(xw + 2 * t2);
        b1 = ld_relaxed_u64(xw + 2 * t2 + 1);
      }
      const bool mine = (a0 & hi_mask) == tag && (a1 & hi_mask) == tag &&
                        (b0 & hi_mask) == tag && (b1 & hi_mask) == tag;
      if (__syncthreads_and(mine)) {
        const double p1 = tid < G ? __longlong_as_double((long long)((a1 << 32) | (a0 & 0xffffffffull))) : 0.0;
        const double p2 = t2 < G ? __longlong_as_double((long long)((b1 << 32) | (b0 & 0xffffffffull))) : 0.0;
        v = p1 + p2;
        done = true;
        break;
      }
      if (__syncthreads_or((it & 7u) == 7u && global_timer_ns() - tw0 > kWaitLimitNs)) break;
    }
    v = block_sum_f64(v, red);                   // a fixed tree: the same sum every launch
    if (tid == 0) {
      if (done) {
        const float g = count > 0 ? (float)(v / (double)count) : 0.0f;
        *gamma_out = g;
        const unsigned long long gb = __float_as_uint(g);
        st_relaxed_u64(gwords, tag | gb);
        st_relaxed_u64(gwords + 1, (epoch & hi_mask) | gb);
      } else {
        record_device_error(DEV_ERR_TIMEOUT);
      }
    }
  }
  if (tid == 0) {
    // gamma is this launch's once the first word carries the low half of the
    // epoch and the second the high half, with equal gamma bits
    const unsigned long long tw0 = global_timer_ns();
    bool done = false;
    uint32_t gb = 0u;
    for (uint32_t it = 0;; ++it) {
      const unsigned long long a = ld_relaxed_u64(gwords), b = ld_relaxed_u64(gwords + 1);
      if ((a & hi_mask) == tag && (b & hi_mask) == (epoch & hi_mask) && (uint32_t)a == (uint32_t)b) {
        gb = (uint32_t)a;
        done = true;
        break;
      }
      if ((it & 15u) == 15u && global_timer_ns() - tw0 > kWaitLimitNs) break;
    }
    if (!done) record_device_error(DEV_ERR_TIMEOUT);
    s_gamma = __uint_as_float(gb);
    xok = done ? 1 : 0;
  }
  __syncthreads();
  if (xok) {
    const float g = s_gamma;
    const bool live = gamma_codes_live(g);
    const uint32_t dcode = ternary_dcode<BF16>(__float_as_uint(ternary_threshold(g)));
    // The 16-byte units of a word are read in the order (k + rot) % UPW, so
    // that the 8 lanes of a 128-bit shared-memory access phase touch 8
    // distinct 16-byte bank groups; the k-th unit read is unit (k + rot) % UPW
    // of the word, and its flags go to that unit's bit positions.
    const int rot = BF16 ? (lane >> 2) & 1 : (lane >> 1) & 3;
    if (kw == wpr) {
      // pass 2 without padding words: packed word q0 + l holds the weights of
      // word l of the run.  Thread t takes l = t, t + 512, ...; the first
      // unstaged one is loaded before the staged ones are coded
      const int nw = (int)(q1 - q0);
      uint32_t* out = reinterpret_cast<uint32_t*>(packed) + q0;
      const uint4* g16 = reinterpret_cast<const uint4*>(gsrc);
      const uint4* s16 = reinterpret_cast<const uint4*>(pk_smem);
      int lg = tid;
      while (lg < ns) lg += kPackFusedThreads;     // this thread's first unstaged word
      uint4 gx[UPW];
      if (lg < nw) {
#pragma unroll
        for (int k = 0; k < UPW; ++k) gx[k] = ld_stream_v4(g16 + (size_t)lg * UPW + ((k + rot) & (UPW - 1)));
      }
      for (int l = tid; l < nw; l += kPackFusedThreads) {
        uint4 x[UPW];
        if (l < ns) {
#pragma unroll
          for (int k = 0; k < UPW; ++k) x[k] = s16[l * UPW + ((k + rot) & (UPW - 1))];
        } else if (l == lg) {
#pragma unroll
          for (int k = 0; k < UPW; ++k) x[k] = gx[k];
        } else {
#pragma unroll
          for (int k = 0; k < UPW; ++k) x[k] = ld_stream_v4(g16 + (size_t)l * UPW + ((k + rot) & (UPW - 1)));
        }
        uint32_t a = 0u, b = 0u;
#pragma unroll
        for (int k = 0; k < UPW; ++k) {
          if (BF16) ternary_flags_bf16(x[k], 2 * ((k + rot) & 1), dcode, a, b);
          else ternary_flags_f32(x[k], (k + rot) & 3, dcode, a, b);
        }
        out[l] = live ? ternary_word_from_flags(a, b) : 0x55555555u;
      }
    } else {
      // pass 2 with padding words (K % 64 != 0): word q0 + tid + 512 j as
      // (row, word of row), kPackWords at a time (loads of the batch's
      // unstaged words in flight together)
      const int st_rows = kPackFusedThreads / wpr, st_words = kPackFusedThreads - st_rows * wpr;
      long long q = q0 + tid;
      long long cur_n = q / wpr;
      int cur_w = (int)(q - cur_n * wpr);
      while (q < q1) {
        uint4 raw[kPackWords][UPW];
        int rown[kPackWords], wordi[kPackWords];
#pragma unroll
        for (int u = 0; u < kPackWords; ++u) {
          rown[u] = -1;
          if (q < q1) {
            rown[u] = (int)cur_n;
            wordi[u] = cur_w;
            if (cur_w < kw) {
              const long long sl = cur_n * kw + cur_w - s0;      // word of this CTA's run
              const uint8_t* src = sl < ns ? pk_smem + sl * WB : gsrc + sl * WB;
#pragma unroll
              for (int j = 0; j < UPW; ++j) {
                const uint8_t* pj = src + 16 * ((j + rot) & (UPW - 1));
                raw[u][j] = sl < ns ? *reinterpret_cast<const uint4*>(pj) : ld_stream_v4(pj);
              }
            }
            q += kPackFusedThreads;
            cur_n += st_rows;
            cur_w += st_words;
            if (cur_w >= wpr) {
              cur_w -= wpr;
              ++cur_n;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < kPackWords; ++u) {
          if (rown[u] < 0) continue;
          uint32_t word = 0x55555555u;              // padding, or gamma 0: code 1 everywhere
          if (wordi[u] < kw && live) {
            uint32_t a = 0u, b = 0u;
#pragma unroll
            for (int k = 0; k < UPW; ++k) {
              if (BF16) ternary_flags_bf16(raw[u][k], 2 * ((k + rot) & 1), dcode, a, b);
              else ternary_flags_f32(raw[u][k], (k + rot) & 3, dcode, a, b);
            }
            word = ternary_word_from_flags(a, b);
          }
          reinterpret_cast<uint32_t*>(packed + (size_t)rown[u] * ldw)[wordi[u]] = word;
        }
      }
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
