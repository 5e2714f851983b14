// ffn_decode.cuh -- the W1.58A8 FFN of one block at decode sizes (1..16
// tokens) in ONE persistent launch, optionally preceded by the attention
// output projection and its residual (the block after attention).
//
// nnterp encyclopedia "bitnet", "The block, in order" and "The MLP gates with
// a squared ReLU":
//   z = post_attention_layernorm(x)                  RMSNorm, then int8 codes
//   m = relu(gate_proj(z))^2 * up_proj(z)            two BitLinears of z
//   y = x + down_proj(ffn_sub_norm(m))                RMSNorm of m, int8 codes
// and "The projections quantize their inputs and weights" for every
// projection (per-token absmax codes, ternary weights, exact integer
// contraction dequantised by gamma / s).
//
// For a few tokens the FFN streams 13 MB of packed weights and does little
// arithmetic; run as four launches it pays four grid ramps and completions.
// Here one cooperative grid (one CTA per SM) does it:
//   P0  warp 0 bulk-copies the CTA's weight rows into shared memory at once:
//       its gate rows, the matching up rows and its slice of down rows, each
//       as 8 sub-blocks of consecutive rows whose shared-memory starts differ
//       by 16 bytes mod 128, so the 8 rows an mma fragment load touches (one
//       per sub-block, same column) fall in 8 different bank quads;
//   P1  every CTA quantises all tokens of x itself (RMSNorm prelude; a row is
//       spread over several warps, its loads all in flight): x is a few KB,
//       so the redundant work costs less than an exchange;
//   P2  gate and up of its features on the tensor cores (mma.sync m16n8k32,
//       u8 weight codes c = t + 1 x s8 activation codes, int32): a 16-row
//       fragment holds 8 gate rows over the same 8 up rows, so one thread
//       holds the gate and up sums of a feature and forms m = relu(g)^2 * u
//       (fp32, the fused epilogue's operations) directly; the warps split K
//       and add their sums with shared-memory atomics (exact in int32);
//   X1  each CTA publishes its fp64 sums of m^2 per token; exchange;
//   P3  every CTA adds the G partial sums in one fixed order (the same fp32
//       mean square, hence the same r, in every CTA), forms xh = (m r) g for
//       its own features and publishes their max |xh| per token; exchange X2;
//   P4  s = 127 / max over the CTAs' maxima (exact in any order); each CTA
//       writes the codes of its own features to the workspace and publishes
//       their code sum per token; exchange X3; every CTA loads all codes;
//   P5  its down rows against those codes (mma.sync again), dequantised,
//       plus the residual x, stored.
// The first exchange of a launch polls one flag per CTA holding a 64-bit
// epoch that is new for every launch (a per-process counter started at a
// random value), so it needs no reset and the workspace no zeroing; CTA 0
// resets the arrival counters of the later exchanges before it publishes its
// flag, and those exchanges poll one counter word.
#pragma once

#include "common.cuh"
#include "gemv.cuh"
#include "quant_act.cuh"

namespace bitnet {

constexpr int kFdThreads = 256;           // 8 warps
constexpr int kFdMaxSlots = 8;            // rows per gate / up sub-block (<= 64 features per CTA)
constexpr int kFdMaxGrid = 256;           // partials / flags slots in the control block
constexpr int kFdRowPad = 16;             // bytes added to every staged code row
constexpr int kFdRegChunks = 8;           // float4 chunks per thread held in the row quantiser
                                          // (24 held every 1-4-token row at once but made the
                                          // phase code ~3x longer: 34 vs 29 us per FFN at M = 1)

// Control block of one persistent launch, in the caller's workspace.
struct FdControl {
  double ss[kFdMaxGrid][16];              // per-CTA sums of m^2, per token
  float mx[kFdMaxGrid][16];               // per-CTA max |xh|, per token
  int cs[kFdMaxGrid][16];                 // per-CTA code sums, per token
  unsigned long long flags[kFdMaxGrid];   // first exchange: epoch flags
  unsigned int ctr[4];                    // later exchanges: arrival counters
};

struct FfnDecodeParams {
  const void* X;               // [M][H] bf16 or fp32
  int x_bf16;
  int M, H, I;
  const uint8_t* Wg;           // [I][ldwH] device-layout packed rows
  const uint8_t* Wu;
  const uint8_t* Wd;           // [H][ldwI]
  const float* gamma_g;
  const float* gamma_u;
  const float* gamma_d;
  const float* pre_gain;       // [H] or null
  const float* sub_gain;       // [I] or null
  float eps;
  void* Y;                     // [M][H], y_bf16 ? bf16 : fp32
  int y_bf16;
  float* hid;                  // [M][I] fp32 m (each CTA its features; for inspection)
  int8_t* hq;                  // [M][I] sub-norm codes (each CTA its features; read back by all)
  float* hs;                   // [M] their scales (CTA 0)
  int32_t* hrs;                // [M] their code sums (CTA 0)
  FdControl* ctl;
  unsigned long long epoch;
  // the block after attention (TAIL kernels only): X is the residual stream
  // x, A the attention output, h = x + o_proj(attn_sub_norm(A)) in fp32
  const void* A;               // [M][H], X's type
  const uint8_t* Wo;           // [H][ldwH]
  const float* gamma_o;
  const float* attn_gain;      // [H] or null
  float* hbuf;                 // [M][H] fp32 h (workspace)
  void* H_out;                 // [M][H] h in Y's type, or null
  int ldwH, ldwI;
  int nf_per, nr_per;          // features / down rows per CTA (the last CTAs fewer)
  int slots;                   // rows per gate / up sub-block: ceil(nf_per / 8)
  int mpad;                    // tokens rounded up to 8
  // shared-memory carve-up (bytes from the 128-aligned base): gate sub-blocks
  // at 0, up at off_u, down (TAIL: o_proj first, then down) at off_d
  int off_u, off_d, off_act;
  int sx_h, sx_i;              // staged code row strides (K + 16: conflict-free fragments)
};

struct FfnDecodeShared {
  int red[kFdMaxSlots * 2 * 32 * 4];    // P2 sums [slot][ntile][lane][4]; P5 reuses it
  float f_hi[2][16], f_lo[2][16];       // dequant factors of x (gate, up) per token
  int rs_x[16];
  float s_x[16];
  float fd_hi[16], fd_lo[16];           // down dequant factors per token
  int rs_m[16];
  float s_m[16];                        // sub-norm scales per token
  float r_m[16];                        // sub-norm 1 / rms per token
  int zr_m[16];                         // all-zero hidden row
  float fo_hi[16], fo_lo[16];           // o_proj dequant factors per token
  int rs_a[16];
  float s_a[16];
  int ok;                               // weights landed / exchanges completed
  int xok;
  __align__(8) uint64_t bar_gu, bar_d, bar_o;
};

// ---- sub-block layout of a CTA's n staged rows (row stride ldw bytes):
// sub-block g (0..7) holds sb_count(n, g) consecutive rows starting at row
// sb_first(n, g), at byte sb_base(n, ldw, g) = 16 g (mod 128).
__host__ __device__ inline int sb_count(int n, int g) { return n / 8 + (g < n % 8 ? 1 : 0); }
__host__ __device__ inline int sb_first(int n, int g) {
  return g * (n / 8) + (g < n % 8 ? g : n % 8);
}
__host__ __device__ inline int sb_span(int n, int ldw, int g) {
  return (sb_count(n, g) * ldw + 128 + 127) & ~127;
}
__host__ __device__ inline int sb_base(int n, int ldw, int g) {
  int b = 0;
  for (int j = 0; j < g; ++j) b += sb_span(n, ldw, j);
  return b + 16 * g;
}
__host__ __device__ inline int sb_bytes(int n, int ldw) { return sb_base(n, ldw, 8) - 16 * 8; }

__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 1-D bulk copy global -> shared, completing on an mbarrier (16-byte aligned
// addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Sub-blocks of rows [row0, row0 + n) of a packed matrix into shared memory
// at `dst` (lane g of the calling warp copies sub-block g).
__device__ __forceinline__ void copy_sub_blocks(uint8_t* dst, const uint8_t* W, int row0, int n,
                                                int ldw, uint64_t* bar, int lane) {
  if (lane < 8) {
    const int cnt = sb_count(n, lane);
    if (cnt > 0)
      bulk_copy_g2s(dst + sb_base(n, ldw, lane),
                    W + (size_t)(row0 + sb_first(n, lane)) * ldw, (uint32_t)(cnt * ldw), bar);
  }
}

// L2-coherent loads of data other CTAs of this grid wrote.
__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_cg_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ double ld_cg_f64(const double* p) {
  double v;
  asm volatile("ld.global.cg.f64 %0, [%1];" : "=d"(v) : "l"(p));
  return v;
}

// Sum over the warp of a double in a fixed xor tree (every lane gets it).
__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max_f32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// int8 code of an already scaled value y (|y| <= 127 (1 + 2^-24)^2): rint
// half-to-even by one fp32 add of 1.5 * 2^23, the code is the sum's low byte.
__device__ __forceinline__ int code_of(float y) {
  return (int)(int8_t)(__float_as_uint(__fadd_rn(y, 12582912.0f)) & 0xffu);
}

template <int KIND>
__device__ __forceinline__ float4 fd_load4(const void* src, size_t elem) {
  if (KIND == 1) {
    const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(src) + elem);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
  } else if (KIND == 2) {
    return ld_cg_f4(reinterpret_cast<const float*>(src) + elem);
  }
  return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(src) + elem);
}

// Codes of the M token rows of an [M][n] activation (RMSNorm prelude, the
// library's arithmetic: mean square accumulated in fp64 from exact squares and
// rounded once, r = 1/sqrt(ms + eps) in fp32, xh = (x r) g, s = 127 / max|xh|,
// q = rint(xh s)) into shared memory rows of `stride` bytes.  Rows past M are
// not written (their mma columns are discarded).  Every thread of the CTA
// calls it.
//   Rows are spread over the warps so that all of them work for any M: with
//   rp rows in flight (1, 2, 4 or 8), a row gets gw = 8 / rp warps, and each
//   of its threads holds up to kFdRegChunks float4 chunks in registers, all
//   loaded before any is used (longer rows are done in batches, reloaded per
//   pass).  A thread keeps four fp64 sums (one per float4 lane: short
//   dependency chains) added in a fixed order; sums and maxima are then
//   combined in a fixed order (warp xor tree, the row's warps in turn), the
//   same in every CTA.
//   KIND 0: fp32 rows, 1: bf16 rows, 2: fp32 rows this grid wrote (loaded
//   from L2).
template <int KIND>
__device__ void fd_quant_rows(const void* src, int M, int n, const float* gain, float eps,
                              int8_t* s_act, int stride, float* s_out, int* rs_out) {
  __shared__ double red_d[8];
  __shared__ float red_f[8];
  __shared__ int red_i[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rp = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;   // rows in flight
  const int gw = 8 / rp;                                      // warps per row
  const int grp = warp / gw, wg = warp - grp * gw;
  const int nc = n / 4;                                       // float4 chunks per row
  const int tstride = 32 * gw;                                // chunk stride of a thread
  const int per = (nc + tstride - 1) / tstride;               // chunks per thread
  const int first = lane + 32 * wg;                           // this thread's first chunk
  const bool fits = per <= kFdRegChunks;
  for (int round = 0; round * rp < M; ++round) {
    const int m = round * rp + grp;
    const bool row = m < M;
    const size_t base = (size_t)(row ? m : 0) * n;
    float4 v[kFdRegChunks];
    // pass 1: sum of squares and max|x|
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
    float xmax = 0.0f;
    for (int b0 = 0; b0 < per; b0 += kFdRegChunks) {
#pragma unroll
      for (int i = 0; i < kFdRegChunks; ++i) {
        const int c = first + (b0 + i) * tstride;
        v[i] = (row && b0 + i < per && c < nc) ? fd_load4<KIND>(src, base + 4 * (size_t)c)
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int i = 0; i < kFdRegChunks; ++i) {
        if (row && b0 + i < per && first + (b0 + i) * tstride < nc) {
          s0 = fma((double)v[i].x, (double)v[i].x, s0);
          s1 = fma((double)v[i].y, (double)v[i].y, s1);
          s2 = fma((double)v[i].z, (double)v[i].z, s2);
          s3 = fma((double)v[i].w, (double)v[i].w, s3);
          xmax = fmaxf(xmax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)),
                                   fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
        }
      }
    }
    double ss = warp_sum_f64((s0 + s1) + (s2 + s3));
    xmax = warp_max_f32(xmax);
    if (lane == 0) { red_d[warp] = ss; red_f[warp] = xmax; }
    __syncthreads();
    ss = 0.0;
    xmax = 0.0f;
    for (int w = 0; w < gw; ++w) {
      ss += red_d[grp * gw + w];
      xmax = fmaxf(xmax, red_f[grp * gw + w]);
    }
    __syncthreads();
    const float ms = (float)(ss / (double)n);
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    // pass 2 (with a gain): max|xh|; without one, max|fl(x r)| = fl(max|x| r)
    float amax;
    if (gain == nullptr) {
      amax = xmax == 0.0f ? 0.0f : __fmul_rn(xmax, r);
    } else {
      amax = 0.0f;
      for (int b0 = 0; b0 < per; b0 += kFdRegChunks) {
        if (!fits) {
#pragma unroll
          for (int i = 0; i < kFdRegChunks; ++i) {
            const int c = first + (b0 + i) * tstride;
            v[i] = (row && b0 + i < per && c < nc) ? fd_load4<KIND>(src, base + 4 * (size_t)c)
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int i = 0; i < kFdRegChunks; ++i) {
          const int c = first + (b0 + i) * tstride;
          if (row && b0 + i < per && c < nc) {
            const float4 g = __ldg(reinterpret_cast<const float4*>(gain) + c);
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(__fmul_rn(__fmul_rn(v[i].x, r), g.x)),
                                           fabsf(__fmul_rn(__fmul_rn(v[i].y, r), g.y))),
                                     fmaxf(fabsf(__fmul_rn(__fmul_rn(v[i].z, r), g.z)),
                                           fabsf(__fmul_rn(__fmul_rn(v[i].w, r), g.w)))));
          }
        }
      }
      amax = warp_max_f32(amax);
      if (lane == 0) red_f[warp] = amax;
      __syncthreads();
      amax = 0.0f;
      for (int w = 0; w < gw; ++w) amax = fmaxf(amax, red_f[grp * gw + w]);
      __syncthreads();
    }
    float s = __fdiv_rn(127.0f, amax);
    const bool zero_row = (amax == 0.0f) || isinf(s);
    if (zero_row) s = 1.0f;
    // pass 3: codes and their sum
    int rsum = 0;
    int8_t* dst = s_act + (size_t)(row ? m : 0) * stride;
    for (int b0 = 0; b0 < per; b0 += kFdRegChunks) {
      if (!fits) {
#pragma unroll
        for (int i = 0; i < kFdRegChunks; ++i) {
          const int c = first + (b0 + i) * tstride;
          v[i] = (row && b0 + i < per && c < nc) ? fd_load4<KIND>(src, base + 4 * (size_t)c)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int i = 0; i < kFdRegChunks; ++i) {
        const int c = first + (b0 + i) * tstride;
        if (row && b0 + i < per && c < nc) {
          uint32_t w = 0u;
          if (!zero_row) {
            const float4 g = gain ? __ldg(reinterpret_cast<const float4*>(gain) + c)
                                  : make_float4(1.f, 1.f, 1.f, 1.f);
            w = pack_codes4(__fmul_rn(__fmul_rn(__fmul_rn(v[i].x, r), g.x), s),
                            __fmul_rn(__fmul_rn(__fmul_rn(v[i].y, r), g.y), s),
                            __fmul_rn(__fmul_rn(__fmul_rn(v[i].z, r), g.z), s),
                            __fmul_rn(__fmul_rn(__fmul_rn(v[i].w, r), g.w), s));
            rsum = __dp4a((int)w, 0x01010101, rsum);
          }
          *reinterpret_cast<uint32_t*>(dst + 4 * c) = w;
        }
      }
    }
    rsum = __reduce_add_sync(0xffffffffu, rsum);
    if (lane == 0) red_i[warp] = rsum;
    __syncthreads();
    if (row && wg == 0 && lane == 0) {
      int t = 0;
      for (int w = 0; w < gw; ++w) t += red_i[grp * gw + w];
      s_out[m] = s;
      rs_out[m] = t;
    }
    __syncthreads();
  }
}

// int32 sums of the CTA's nr staged rows (sub-block layout, stride ldw)
// against the staged codes (stride sx) over K inputs, added into
// red[(i * 2 + t) * 32 + lane][4]: row tile i <= 1 holds slots 2i (fragment
// rows 0..7, one per sub-block) and 2i + 1 (rows 8..15) of the sub-blocks,
// token tile t <= 1; the 8 warps split the K steps of 32.
__device__ __forceinline__ void fd_contract_rows(const uint8_t* s_w, int ldw, int nr,
                                                 const int8_t* s_x, int sx, int K, int ntile,
                                                 int* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, c4 = lane & 3;
  const int steps = K / 32;
  const int s_lo = warp * steps / 8, s_hi = (warp + 1) * steps / 8;
  const int cmax = sb_count(nr, 0);                  // slots of the largest sub-block
  const int cnt = sb_count(nr, g8);
  const int clast = cnt > 0 ? cnt - 1 : 0;           // slots past cnt read a valid row
  const uint8_t* wb = s_w + sb_base(nr, ldw, g8);
  int acc[2][2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][t][e] = 0;
  for (int s = s_lo; s < s_hi; ++s) {
    uint32_t bf[2][2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (t < ntile) {
        const int8_t* xr = s_x + (size_t)(8 * t + g8) * sx + 32 * s + 4 * c4;
        bf[t][0] = *reinterpret_cast<const uint32_t*>(xr);
        bf[t][1] = *reinterpret_cast<const uint32_t*>(xr + 16);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (2 * i < cmax) {
        const uint2 lo = *reinterpret_cast<const uint2*>(wb + (size_t)min(2 * i, clast) * ldw + 8 * s);
        const uint2 hi =
            *reinterpret_cast<const uint2*>(wb + (size_t)min(2 * i + 1, clast) * ldw + 8 * s);
        const uint32_t a0 = (lo.x >> (2 * c4)) & 0x03030303u;
        const uint32_t a2 = (lo.y >> (2 * c4)) & 0x03030303u;
        const uint32_t a1 = (hi.x >> (2 * c4)) & 0x03030303u;
        const uint32_t a3 = (hi.y >> (2 * c4)) & 0x03030303u;
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (t < ntile) mma_u8s8_16832(acc[i][t], a0, a1, a2, a3, bf[t][0], bf[t][1]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int t = 0; t < 2; ++t)
      if (2 * i < cmax && t < ntile)
#pragma unroll
        for (int e = 0; e < 4; ++e) atomicAdd(&red[((i * 2 + t) * 32 + lane) * 4 + e], acc[i][t][e]);
}

// Row index (within the CTA's nr rows) of output element (row tile i, half,
// lane) of fd_contract_rows, or -1.
__device__ __forceinline__ int fd_contract_row(int nr, int i, int half, int lane) {
  const int g = lane >> 2, slot = 2 * i + half;
  return slot < sb_count(nr, g) ? sb_first(nr, g) + slot : -1;
}

template <bool TAIL>
__global__ void __launch_bounds__(kFdThreads, 1) ffn_decode_kernel(FfnDecodeParams p) {
  extern __shared__ uint8_t fd_smem_raw[];
  __shared__ FfnDecodeShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(fd_smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* s_g = smem;                      // gate sub-blocks (ldwH rows)
  uint8_t* s_u = smem + p.off_u;            // up sub-blocks
  uint8_t* s_d = smem + p.off_d;            // down sub-blocks (ldwI rows); TAIL: o_proj first
  int8_t* s_act = reinterpret_cast<int8_t*>(smem + p.off_act);   // [mpad][sx_h or sx_i]
  FdControl* ctl = p.ctl;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, c4 = lane & 3;          // mma fragment coordinates
  const int G = gridDim.x, b = blockIdx.x;
  // this CTA's features [f0, f0 + nf) and output rows [n0, n0 + nr) (down
  // rows, and o_proj rows for TAIL)
  const int f0 = b * p.nf_per;
  const int nf = max(0, min(p.nf_per, p.I - f0));
  const int n0 = b * p.nr_per;
  const int nr = max(0, min(p.nr_per, p.H - n0));
  const int M = p.M;
  const int ntile = p.mpad / 8;

  // ---- P0: weight rows -> shared memory (warp 0: lane g copies sub-block g)
  if (threadIdx.x == 0) {
    mbar_init(&sh.bar_gu, 1);
    mbar_init(&sh.bar_d, 1);
    mbar_init(&sh.bar_o, 1);
    fence_barrier_init();
    sh.ok = 1;
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {
      if (TAIL) mbar_arrive_expect_tx(&sh.bar_o, (uint32_t)(nr * p.ldwH));
      mbar_arrive_expect_tx(&sh.bar_gu, (uint32_t)(2 * nf * p.ldwH));
      if (!TAIL) mbar_arrive_expect_tx(&sh.bar_d, (uint32_t)(nr * p.ldwI));
    }
    __syncwarp();
    if (TAIL) copy_sub_blocks(s_d, p.Wo, n0, nr, p.ldwH, &sh.bar_o, lane);   // needed first
    copy_sub_blocks(s_g, p.Wg, f0, nf, p.ldwH, &sh.bar_gu, lane);
    copy_sub_blocks(s_u, p.Wu, f0, nf, p.ldwH, &sh.bar_gu, lane);
    if (!TAIL) copy_sub_blocks(s_d, p.Wd, n0, nr, p.ldwI, &sh.bar_d, lane);
  }

  // ---- TAIL: h = x + o_proj(attn_sub_norm(A)) for this CTA's rows, then
  // the first exchange; every CTA then quantises all of h
  if constexpr (TAIL) {
    if (p.x_bf16)
      fd_quant_rows<1>(p.A, M, p.H, p.attn_gain, p.eps, s_act, p.sx_h, sh.s_a, sh.rs_a);
    else
      fd_quant_rows<0>(p.A, M, p.H, p.attn_gain, p.eps, s_act, p.sx_h, sh.s_a, sh.rs_a);
    for (int i = threadIdx.x; i < 2 * 2 * 32 * 4; i += kFdThreads) sh.red[i] = 0;
    __syncthreads();
    if (threadIdx.x < M) dequant_factor(__ldg(p.gamma_o), sh.s_a[threadIdx.x],
                                        sh.fo_hi[threadIdx.x], sh.fo_lo[threadIdx.x]);
    if (!mbar_wait(&sh.bar_o, 0, nullptr) && lane == 0) sh.ok = 0;
    fd_contract_rows(s_d, p.ldwH, nr, s_act, p.sx_h, p.H, ntile, sh.red);
    __syncthreads();
    // the o_proj rows are read: the down rows go to the same place
    if (warp == 0) {
      if (lane == 0) {
        fence_proxy_async_shared();
        mbar_arrive_expect_tx(&sh.bar_d, (uint32_t)(nr * p.ldwI));
      }
      __syncwarp();
      if (lane < 8) fence_proxy_async_shared();
      copy_sub_blocks(s_d, p.Wd, n0, nr, p.ldwI, &sh.bar_d, lane);
    }
    if (threadIdx.x < 2 * 2 * 32) {
      const int idx = threadIdx.x;
      const int i = idx >> 6, t = (idx >> 5) & 1, ln = idx & 31;
      if (t < ntile) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int r = fd_contract_row(nr, i, half, ln);
          if (r < 0) continue;
          const int n = n0 + r;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int m = 8 * t + 2 * (ln & 3) + e;
            if (m >= M) continue;
            const int acc = sh.red[idx * 4 + 2 * half + e] - sh.rs_a[m];
            const float o = dequant_dw(acc, sh.fo_hi[m], sh.fo_lo[m]);
            const size_t at = (size_t)m * p.H + n;
            const float x = p.x_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.X)[at])
                                     : reinterpret_cast<const float*>(p.X)[at];
            const float h = __fadd_rn(x, o);
            p.hbuf[at] = h;
            if (p.H_out != nullptr) {
              if (p.y_bf16)
                reinterpret_cast<__nv_bfloat16*>(p.H_out)[at] = __float2bfloat16_rn(h);
              else
                reinterpret_cast<float*>(p.H_out)[at] = h;
            }
          }
        }
      }
    }
    if (!grid_exchange(ctl->flags, p.epoch, &sh.xok, ctl->ctr, 4) && threadIdx.x == 0) sh.ok = 0;
    fd_quant_rows<2>(p.hbuf, M, p.H, p.pre_gain, p.eps, s_act, p.sx_h, sh.s_x, sh.rs_x);
  } else {
    // ---- P1: codes of x (RMSNorm prelude), every token, into s_act
    if (p.x_bf16)
      fd_quant_rows<1>(p.X, M, p.H, p.pre_gain, p.eps, s_act, p.sx_h, sh.s_x, sh.rs_x);
    else
      fd_quant_rows<0>(p.X, M, p.H, p.pre_gain, p.eps, s_act, p.sx_h, sh.s_x, sh.rs_x);
  }
  __syncthreads();
  if (threadIdx.x < M) {
    const int m = threadIdx.x;
    dequant_factor(__ldg(p.gamma_g), sh.s_x[m], sh.f_hi[0][m], sh.f_lo[0][m]);
    dequant_factor(__ldg(p.gamma_u), sh.s_x[m], sh.f_hi[1][m], sh.f_lo[1][m]);
  }
  for (int i = threadIdx.x; i < kFdMaxSlots * 2 * 32 * 4; i += kFdThreads) sh.red[i] = 0;
  __syncthreads();

  // ---- P2: gate / up sums of this CTA's features (warps split K).  Fragment
  // rows 0..7 are the gate rows of one feature per sub-block (slot j), rows
  // 8..15 the up rows of the same features.
  {
    const bool landed = mbar_wait(&sh.bar_gu, 0, nullptr);
    if (!landed && lane == 0) sh.ok = 0;
    const int cnt = sb_count(nf, g8);
    const int clast = cnt > 0 ? cnt - 1 : 0;         // slots past cnt read a valid row
    const int sbase = sb_base(nf, p.ldwH, g8);
    const uint8_t* gb = s_g + sbase;
    const uint8_t* ub = s_u + sbase;
    const int steps = p.H / 32;
    const int s_lo = warp * steps / 8, s_hi = (warp + 1) * steps / 8;
    int acc[kFdMaxSlots][2][4];
#pragma unroll
    for (int j = 0; j < kFdMaxSlots; ++j)
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][t][e] = 0;
    for (int s = s_lo; s < s_hi; ++s) {
      uint32_t bf[2][2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t < ntile) {
          const int8_t* xr = s_act + (size_t)(8 * t + g8) * p.sx_h + 32 * s + 4 * c4;
          bf[t][0] = *reinterpret_cast<const uint32_t*>(xr);
          bf[t][1] = *reinterpret_cast<const uint32_t*>(xr + 16);
        }
      }
#pragma unroll
      for (int j = 0; j < kFdMaxSlots; ++j) {
        if (j < p.slots) {
          const size_t off = (size_t)min(j, clast) * p.ldwH + 8 * s;
          const uint2 lo = *reinterpret_cast<const uint2*>(gb + off);       // gate row
          const uint2 hi = *reinterpret_cast<const uint2*>(ub + off);       // up row
          const uint32_t a0 = (lo.x >> (2 * c4)) & 0x03030303u;
          const uint32_t a2 = (lo.y >> (2 * c4)) & 0x03030303u;
          const uint32_t a1 = (hi.x >> (2 * c4)) & 0x03030303u;
          const uint32_t a3 = (hi.y >> (2 * c4)) & 0x03030303u;
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if (t < ntile) mma_u8s8_16832(acc[j][t], a0, a1, a2, a3, bf[t][0], bf[t][1]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kFdMaxSlots; ++j)
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (j < p.slots && t < ntile)
#pragma unroll
          for (int e = 0; e < 4; ++e) atomicAdd(&sh.red[((j * 2 + t) * 32 + lane) * 4 + e], acc[j][t][e]);
  }
  __syncthreads();
  // m = relu(g)^2 * u for (feature, token): thread (slot j, tile t, lane)
  // holds gate sums of the feature in slot j of sub-block lane / 4 for tokens
  // 8t + 2 (lane % 4) + {0, 1} in red[.][0..1] and the up sums in red[.][2..3]
  float* m_loc = reinterpret_cast<float*>(sh.red);   // reused below: [16][64] after a barrier
  float mvals[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  int mf[2] = {-1, -1};
  int mm[2][2];
  for (int it = 0; it < 2; ++it) {
    const int idx = threadIdx.x + it * kFdThreads;     // (j * 2 + t) * 32 + lane
    const int jt = idx >> 5, ln = idx & 31;
    const int j = jt >> 1, t = jt & 1;
    const int g = ln >> 2;
    if (j >= p.slots || t >= ntile || j >= sb_count(nf, g)) continue;
    const int f = sb_first(nf, g) + j;
    mf[it] = f;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int m = 8 * t + 2 * (ln & 3) + e;
      mm[it][e] = m;
      if (m >= M) continue;
      const int dg = sh.red[idx * 4 + e] - sh.rs_x[m];
      const int du = sh.red[idx * 4 + 2 + e] - sh.rs_x[m];
      const float gv = dequant_dw(dg, sh.f_hi[0][m], sh.f_lo[0][m]);
      const float uv = dequant_dw(du, sh.f_hi[1][m], sh.f_lo[1][m]);
      mvals[it][e] = __fmul_rn(gv > 0.0f ? __fmul_rn(gv, gv) : 0.0f, uv);
    }
  }
  __syncthreads();                                    // red[] is read: reuse it as m_loc
  for (int it = 0; it < 2; ++it) {
    if (mf[it] < 0) continue;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int m = mm[it][e];
      if (m < M) {
        m_loc[m * 64 + mf[it]] = mvals[it][e];
        p.hid[(size_t)m * p.I + f0 + mf[it]] = mvals[it][e];
      }
    }
  }
  __syncthreads();
  // per token: fp64 sum of m^2 over this CTA's features in a fixed order
  for (int m = warp; m < M; m += kFdThreads / 32) {
    double v = 0.0;
    for (int f = lane; f < nf; f += 32) {
      const double d = (double)m_loc[m * 64 + f];
      v = fma(d, d, v);
    }
    v = warp_sum_f64(v);
    if (lane == 0) ctl->ss[b][m] = v;
  }

  // ---- X1: the sums of m^2
  if (TAIL) {
    if (!grid_count_exchange(&ctl->ctr[0], (unsigned)G, &sh.xok) && threadIdx.x == 0) sh.ok = 0;
  } else {
    if (!grid_exchange(ctl->flags, p.epoch, &sh.xok, ctl->ctr, 4) && threadIdx.x == 0) sh.ok = 0;
  }

  // ---- P3: r per token (the G partial sums in one fixed order: lanes take
  // every 32nd CTA in turn, then the warp's xor tree), then xh of this CTA's
  // features and their max
  for (int m = warp; m < M; m += kFdThreads / 32) {
    double v = 0.0;
    for (int i = lane; i < G; i += 32) v += ld_cg_f64(&ctl->ss[i][m]);
    v = warp_sum_f64(v);
    if (lane == 0) {
      const float ms = (float)(v / (double)p.I);
      sh.r_m[m] = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.eps)));
    }
  }
  __syncthreads();
  for (int m = warp; m < M; m += kFdThreads / 32) {
    const float r = sh.r_m[m];
    float amax = 0.0f;
    for (int f = lane; f < nf; f += 32) {
      const float g = p.sub_gain ? __ldg(p.sub_gain + f0 + f) : 1.0f;
      const float xh = __fmul_rn(__fmul_rn(m_loc[m * 64 + f], r), g);
      m_loc[m * 64 + f] = xh;
      amax = fmaxf(amax, fabsf(xh));
    }
    amax = warp_max_f32(amax);
    if (lane == 0) ctl->mx[b][m] = amax;
  }

  // ---- X2: the maxima
  if (!grid_count_exchange(&ctl->ctr[TAIL ? 1 : 0], (unsigned)G, &sh.xok) && threadIdx.x == 0)
    sh.ok = 0;

  // ---- P4: s per token, codes of this CTA's features -> workspace
  for (int m = warp; m < M; m += kFdThreads / 32) {
    float amax = 0.0f;
    for (int i = lane; i < G; i += 32) amax = fmaxf(amax, __ldcg(&ctl->mx[i][m]));
    amax = warp_max_f32(amax);
    float s = __fdiv_rn(127.0f, amax);
    const bool zero_row = (amax == 0.0f) || isinf(s);
    if (zero_row) s = 1.0f;
    int csum = 0;
    for (int f = lane; f < nf; f += 32) {
      const int q = zero_row ? 0 : code_of(__fmul_rn(m_loc[m * 64 + f], s));
      p.hq[(size_t)m * p.I + f0 + f] = (int8_t)q;
      csum += q;
    }
    csum = __reduce_add_sync(0xffffffffu, csum);
    if (lane == 0) {
      ctl->cs[b][m] = csum;
      sh.s_m[m] = s;
    }
  }

  // ---- X3: the codes
  if (!grid_count_exchange(&ctl->ctr[TAIL ? 2 : 1], (unsigned)G, &sh.xok) && threadIdx.x == 0)
    sh.ok = 0;

  // every CTA: code sums, and all codes into s_act (16-byte loads from L2,
  // four in flight per thread)
  for (int m = warp; m < M; m += kFdThreads / 32) {
    int v = 0;
    for (int i = lane; i < G; i += 32) v += __ldcg(&ctl->cs[i][m]);
    v = __reduce_add_sync(0xffffffffu, v);
    if (lane == 0) sh.rs_m[m] = v;
  }
  {
    const int per_row = p.I / 16;
    const int total = M * per_row;
    for (int base = threadIdx.x; base < total; base += 4 * kFdThreads) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = base + u * kFdThreads;
        if (idx < total)
          v[u] = ld_cg_u4(p.hq + (size_t)(idx / per_row) * p.I + 16 * (idx % per_row));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = base + u * kFdThreads;
        if (idx < total)
          *reinterpret_cast<uint4*>(s_act + (size_t)(idx / per_row) * p.sx_i + 16 * (idx % per_row)) = v[u];
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < M) {
    const int m = threadIdx.x;
    dequant_factor(__ldg(p.gamma_d), sh.s_m[m], sh.fd_hi[m], sh.fd_lo[m]);
    if (b == 0) {
      p.hs[m] = sh.s_m[m];
      p.hrs[m] = sh.rs_m[m];
    }
  }
  for (int i = threadIdx.x; i < 2 * 2 * 32 * 4; i += kFdThreads) sh.red[i] = 0;
  __syncthreads();

  // ---- P5: down rows of this CTA (warps split K), residual, store
  if (!mbar_wait(&sh.bar_d, 0, nullptr) && lane == 0) sh.ok = 0;
  fd_contract_rows(s_d, p.ldwI, nr, s_act, p.sx_i, p.I, ntile, sh.red);
  __syncthreads();
  if (threadIdx.x < 2 * 2 * 32) {
    // thread (row tile i, token tile t, lane): slots 2i and 2i + 1 of sub-block
    // lane / 4, tokens 8 t + 2 (lane % 4) + {0, 1}
    const int idx = threadIdx.x;
    const int i = idx >> 6, t = (idx >> 5) & 1, ln = idx & 31;
    if (t < ntile && sh.ok) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = fd_contract_row(nr, i, half, ln);
        if (r < 0) continue;
        const int n = n0 + r;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int m = 8 * t + 2 * (ln & 3) + e;
          if (m >= M) continue;
          const int acc = sh.red[idx * 4 + 2 * half + e] - sh.rs_m[m];
          const float y = dequant_dw(acc, sh.fd_hi[m], sh.fd_lo[m]);
          const size_t o = (size_t)m * p.H + n;
          if (TAIL) {                                 // residual: the fp32 h
            const float out = __fadd_rn(__ldcg(p.hbuf + o), y);
            if (p.y_bf16)
              reinterpret_cast<__nv_bfloat16*>(p.Y)[o] = __float2bfloat16_rn(out);
            else
              reinterpret_cast<float*>(p.Y)[o] = out;
          } else {
            store_value(p.Y, p.X, o, y, p.y_bf16 ? OUT_BF16 : OUT_F32, EPI_RESIDUAL);
          }
        }
      }
    }
  }
}

}  // namespace bitnet
