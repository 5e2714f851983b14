// gemv.cuh -- decode BitLinear (M <= 16 tokens): int8 activations x packed
// ternary weights -> int32 -> dequantised output.
//
// nnterp encyclopedia "bitnet", "The projections quantize their inputs and
// weights": the projection output equals the linear map of the rounded input
// by the ternarised weight exactly; "BitNet b1.58 2B4T", "How to Use": the
// efficiency needs specialised kernels.
//
// HBM-bound on the packed weights (0.25 byte per weight).  Persistent CTAs
// stage the M activation rows once in shared memory; each warp then streams
// R weight rows at a time with 128-bit non-allocating loads, expands every
// 32-bit word of 16 codes into four words of byte codes with two ALU ops each,
// and multiplies them against the activation bytes with dp4a (unsigned codes
// c = t + 1 times signed activations).  The sum over k of q * c minus the
// token's sum of q is the exact int32 contraction with t.
#pragma once

#include "common.cuh"

namespace bitnet {

enum { OUT_F32 = 0, OUT_BF16 = 1, OUT_I32 = 2 };
enum { EPI_RESIDUAL = 0x10, EPI_SILU = 0x20, LAUNCH_PDL = 0x100, LAUNCH_PDL_INPUTS = 0x200 };
// Internal launch flag (never taken from a caller): the streaming decode
// kernel lets its dependents launch at its start even when it waits for its
// predecessor before loading activations (see gemv_stream_kernel).
enum { LAUNCH_TRIGGER_EARLY = 0x1000 };

constexpr int kMaxSegments = 4;

struct LinearParams {
  const int8_t* Xq;
  const float* xs;
  const int32_t* xrs;
  const uint8_t* W;
  const float* gamma;
  int M, N, K, ldw;
  void* Y;
  int out_type;
  int flags;
  const void* resid;
  // Projections sharing the activations (the decode kernels run them in one
  // launch): projection i owns rows [seg_row0[i], seg_row0[i + 1]) of the
  // concatenated output rows, N above being their total.  A single
  // projection is the table {0, N} with W, gamma, Y.
  int nseg;
  int seg_row0[kMaxSegments + 1];
  const uint8_t* seg_W[kMaxSegments];
  const float* seg_gamma[kMaxSegments];
  void* seg_Y[kMaxSegments];
  // prefill GEMM: the preceding work does not write the packed weights, so
  // the first stages' weight tiles may load before the dependency wait
  int w_early = 0;
};

__host__ __device__ inline void single_segment(LinearParams& p) {
  p.nseg = 1;
  p.seg_row0[0] = 0;
  p.seg_row0[1] = p.N;
  p.seg_W[0] = p.W;
  p.seg_gamma[0] = p.gamma;
  p.seg_Y[0] = p.Y;
}

// Projection of concatenated row n, and its row within that projection.
__device__ __forceinline__ int segment_of(const LinearParams& p, int n, int& local) {
  int s = 0;
#pragma unroll
  for (int i = 1; i < kMaxSegments; ++i)
    if (i < p.nseg && n >= p.seg_row0[i]) s = i;
  local = n - p.seg_row0[s];
  return s;
}

// Exact int -> float for |v| < 2^22 with two ALU/FMA ops (no conversion
// unit): place v in the mantissa of 1.5 * 2^23 and subtract 1.5 * 2^23.
__device__ __forceinline__ float int_to_float_exact(int v) {
  return __fsub_rn(__int_as_float(0x4B400000 + v), 12582912.0f);
}

// y = v * (f_hi + f_lo), where f_hi + f_lo is gamma / s to about 2^-48
// relative: one FMA adds the exact product v * f_hi to the rounded small term
// v * f_lo (|f_lo| <= 2^-24 f_hi, so that term's rounding error is ~2^-48 of
// the result), and its one rounding gives the correctly rounded fp32 of
// v * gamma / s except when that value lies within ~2^-46 of an fp32
// midpoint.  The accumulator |v| <= 128 * K <= 2^21 is exact in fp32.
__device__ __forceinline__ float dequant_dw(int v, float f_hi, float f_lo) {
  const float a = int_to_float_exact(v);
  return __fmaf_rn(a, f_hi, __fmul_rn(a, f_lo));
}

// Split gamma / s into an fp32 head and tail: the head is the correctly
// rounded quotient, the remainder gamma - head * s is exact in fp32 (one FMA),
// and the tail is that remainder divided by s, so head + tail equals gamma / s
// to about 2^-48 relative.  Only fp32 division and FMA (no fp64 unit).
__device__ __forceinline__ void dequant_factor(float gamma, float s, float& f_hi, float& f_lo) {
  f_hi = __fdiv_rn(gamma, s);
  const float r = __fmaf_rn(-f_hi, s, gamma);
  f_lo = __fdiv_rn(r, s);
}

// Epilogue tail shared by the decode and prefill kernels: fp32 value ->
// optional SiLU / residual -> stored element.
__device__ __forceinline__ void store_value(void* Y, const void* resid, size_t idx, float y,
                                            int out_type, int flags) {
  if (flags & EPI_SILU) {
    y = silu_f32(y);
  }
  if (out_type == OUT_BF16) {
    if (flags & EPI_RESIDUAL) {
      const float r = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(resid)[idx]);
      y = __fadd_rn(r, y);
    }
    reinterpret_cast<__nv_bfloat16*>(Y)[idx] = __float2bfloat16_rn(y);
  } else {
    if (flags & EPI_RESIDUAL) y = __fadd_rn(reinterpret_cast<const float*>(resid)[idx], y);
    reinterpret_cast<float*>(Y)[idx] = y;
  }
}

constexpr int kGemvThreads = 256;
constexpr int kGemvRows = 2;   // weight rows per warp task

template <int MT>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(LinearParams p) {
  extern __shared__ uint4 gemv_smem[];          // [MT][ldw / 4] activation codes (16 B units)
  __shared__ float2 tok_f[MT];
  __shared__ int tok_rs[MT];

  const int chunks = p.ldw / 16;                // 16-byte packed chunks (64 weights) per row
  const int qv = chunks * 4;                    // 16-byte activation units per row
  for (int i = threadIdx.x; i < MT * qv; i += blockDim.x) {
    const int m = i / qv, c = i % qv, k0 = 16 * c;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (m < p.M && k0 < p.K) v = *reinterpret_cast<const uint4*>(p.Xq + (size_t)m * p.K + k0);
    gemv_smem[i] = v;
  }
  if (threadIdx.x < MT) {
    const int m = threadIdx.x;
    float2 f = make_float2(0.0f, 0.0f);
    int rs = 0;
    if (m < p.M) {
      dequant_factor(__ldg(p.gamma), p.xs[m], f.x, f.y);
      rs = p.xrs[m];
    }
    tok_f[m] = f;
    tok_rs[m] = rs;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  for (int n0 = (blockIdx.x * nwarps + warp) * kGemvRows; n0 < p.N;
       n0 += gridDim.x * nwarps * kGemvRows) {
    int acc[kGemvRows][MT];
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0;

#pragma unroll
    for (int r = 0; r < kGemvRows; ++r) {
      const int n = n0 + r;
      if (n < p.N) {
        const uint8_t* wrow = p.W + (size_t)n * p.ldw;
        for (int c = lane; c < chunks; c += 32) {
          const uint4 w = ld_stream_v4(wrow + 16 * c);
          uint32_t e[16];
          expand_codes(w.x, e[0], e[1], e[2], e[3]);
          expand_codes(w.y, e[4], e[5], e[6], e[7]);
          expand_codes(w.z, e[8], e[9], e[10], e[11]);
          expand_codes(w.w, e[12], e[13], e[14], e[15]);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const uint4* qp = gemv_smem + m * qv + 4 * c;
            const uint4 q0 = qp[0], q1 = qp[1], q2 = qp[2], q3 = qp[3];
            int a = acc[r][m];
            a = dp4a_us(e[0], q0.x, a);  a = dp4a_us(e[1], q0.y, a);
            a = dp4a_us(e[2], q0.z, a);  a = dp4a_us(e[3], q0.w, a);
            a = dp4a_us(e[4], q1.x, a);  a = dp4a_us(e[5], q1.y, a);
            a = dp4a_us(e[6], q1.z, a);  a = dp4a_us(e[7], q1.w, a);
            a = dp4a_us(e[8], q2.x, a);  a = dp4a_us(e[9], q2.y, a);
            a = dp4a_us(e[10], q2.z, a); a = dp4a_us(e[11], q2.w, a);
            a = dp4a_us(e[12], q3.x, a); a = dp4a_us(e[13], q3.y, a);
            a = dp4a_us(e[14], q3.z, a); a = dp4a_us(e[15], q3.w, a);
            acc[r][m] = a;
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        int v = acc[r][m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        acc[r][m] = v;
      }
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int n = n0 + r;
        if (lane == ((r * MT + m) & 31) && m < p.M && n < p.N) {
          const size_t idx = (size_t)m * p.N + n;
          const int yint = acc[r][m] - tok_rs[m];
          if (p.out_type == OUT_I32)
            reinterpret_cast<int32_t*>(p.Y)[idx] = yint;
          else
            store_value(p.Y, p.resid, idx, dequant_dw(yint, tok_f[m].x, tok_f[m].y), p.out_type,
                        p.flags);
        }
      }
  }
}

// ---------------------------------------------------------------------------
// Streaming decode for 1..2 tokens (dp4a on the CUDA cores, no tensor memory,
// no cluster) in dependent calls (independent calls, and 3-8 tokens on small
// matrices, take gemv_flat_kernel below).  A warp owns G = 32 / L consecutive
// weight rows, L lanes per row: lane (g, sub) takes chunks sub, sub + L,
// sub + 2L, ... (16 bytes, 64 weights each) of row g, at most J of them, all
// loaded into registers before anything waits, so each lane adds into one
// sum per token and a row's sum is an L-lane butterfly (no per-chunk row
// bookkeeping: a dependent 1-token 4.4 MB call 3.34 -> 2.56 us against lanes
// spread over several rows).  Activation codes are staged in shared memory
// (K a multiple of 64) while the weights land; the lanes of different row
// groups read the same chunks' codes.  The weights (and gamma) are read
// before griddepcontrol.wait (the caller's LAUNCH_PDL statement covers them);
// with LAUNCH_PDL_INPUTS the activations and the whole contraction also
// precede it, and only the output stores wait.  A dependent call (LAUNCH_PDL
// without _INPUTS) lets the next grid launch only after its own wait: in a
// chain of dependent calls that bounds the look-ahead to one call, whose
// weight loads then do not queue in front of the current call's;
// LAUNCH_TRIGGER_EARLY keeps the trigger at the start.
template <int MT, int J>
__global__ void __launch_bounds__(256) gemv_stream_kernel(LinearParams p, int L) {
  // shared memory: the activation codes as [MT][4][C] 16-byte units: unit u
  // of a token row (its inputs 16u .. 16u + 15) sits in plane u % 4 at index
  // u / 4, so lanes holding consecutive chunks read consecutive 16-byte words
  extern __shared__ uint4 gs_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = p.ldw / 16;                    // packed chunks per row
  const int G = 32 / L;                        // rows per warp
  const int nb0 = blockIdx.x * (int)(blockDim.x >> 5) * G;
  const int g = lane / L, sub = lane - g * L;
  const int n = nb0 + warp * G + g;            // this lane's row
  const bool row_ok = n < p.N;
  uint4* s_x = gs_smem;
  const bool inputs_ready = (p.flags & LAUNCH_PDL_INPUTS) != 0;
  const bool trigger_early = inputs_ready || (p.flags & LAUNCH_TRIGGER_EARLY) != 0;
  if (trigger_early) grid_launch_dependents();

  // 1. the weights
  int nl = 0, sg = 0;
  if (row_ok) sg = segment_of(p, n, nl);
  uint4 w[J];
  const uint8_t* src = p.seg_W[sg] + (size_t)nl * p.ldw;
#pragma unroll
  for (int k = 0; k < J; ++k) {
    const int c = sub + L * k;
    w[k] = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);   // t = 0
    if (row_ok && c < C) w[k] = ld_stream_v4(src + 16 * c);
  }
  // the weight scale of this lane's row, part of the packed weights: fetched
  // before any wait
  const float gam = row_ok ? __ldg(p.seg_gamma[sg]) : 0.0f;

  // 2. activation codes, token scales and code sums
  if (!inputs_ready) {
    grid_dependency_wait();
    if (!trigger_early) grid_launch_dependents();
  }
  const int units = p.K / 16;
  for (int i = threadIdx.x; i < MT * units; i += blockDim.x) {
    const int m = i / units, u = i - m * units;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (m < p.M) v = *reinterpret_cast<const uint4*>(p.Xq + (size_t)m * p.K + 16 * u);
    s_x[(m * 4 + (u & 3)) * C + (u >> 2)] = v;
  }
  float xs_m[MT];
  int xrs_m[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    xs_m[m] = m < p.M ? p.xs[m] : 1.0f;
    xrs_m[m] = m < p.M ? p.xrs[m] : 0;
  }
  __syncthreads();

  // 3. unsigned codes x signed activations.  Word u of a chunk holds weight
  // 16u + 4i + j at byte j, bits 2i; masking it with 0x03030303 << 2i (no
  // shift) leaves 4^i times the codes of weights 16u + 4i .. 16u + 4i + 3, so
  // the dp4a chain A_i of mask i carries a factor 4^i, removed once per
  // chunk: A_0 + A_1 / 4 + A_2 / 16 + A_3 / 64, exact (each A_i is a multiple
  // of 4^i; |A_i| < 2^19).
  int acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0;
#pragma unroll
  for (int k = 0; k < J; ++k) {
    const int c = sub + L * k;
    if (row_ok && c < C) {
      const uint4 wj = w[k];
      const uint32_t wv[4] = {wj.x, wj.y, wj.z, wj.w};
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4* qp = s_x + m * 4 * C + c;           // 64 activation codes
        const uint4 qv[4] = {qp[0], qp[C], qp[2 * C], qp[3 * C]};
        int A[4] = {0, 0, 0, 0};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t q4[4] = {qv[u].x, qv[u].y, qv[u].z, qv[u].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) A[i] = dp4a_us(wv[u] & (0x03030303u << (2 * i)), q4[i], A[i]);
        }
        acc[m] += A[0] + (A[1] >> 2) + (A[2] >> 4) + (A[3] >> 6);
      }
    }
  }

  // 4. row sums over the row's L lanes (butterfly: every lane of the group
  // ends with them); lane sub of the group stores tokens m = sub, sub + L, ...
#pragma unroll
  for (int m = 0; m < MT; ++m)
    for (int o = L >> 1; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
  if (inputs_ready) grid_dependency_wait();    // Y may still be read or written before
  if (!row_ok) return;
  const int Ns = p.seg_row0[sg + 1] - p.seg_row0[sg];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if (m % L != sub || m >= p.M) continue;
    const int yint = acc[m] - xrs_m[m];
    const size_t idx = (size_t)m * Ns + nl;
    if (p.out_type == OUT_I32) {
      reinterpret_cast<int32_t*>(p.seg_Y[sg])[idx] = yint;
    } else {
      float fh, fl;
      dequant_factor(gam, xs_m[m], fh, fl);
      store_value(p.seg_Y[sg], p.resid, idx, dequant_dw(yint, fh, fl), p.out_type, p.flags);
    }
  }
}

// Streaming decode with a warp's chunks spread flat over its rows (chunk
// f = lane + 32 j of the warp's R rows), for independent calls
// (LAUNCH_PDL_INPUTS) and for 3-8 tokens on small matrices; the row-group
// kernel above takes the rest.  Measured on the 1-token shapes, this layout
// streams independent calls faster (4.4 MB: 1.27 / 1.43 against 1.49 / 1.74
// us; 1.6 MB: 0.87 against 1.13 us; q/k/v 2.5 MB: 1.05 against 1.67 us) and
// the row groups serve dependent calls better (4.4 MB: 2.56 / 3.07 against
// 3.34 / 3.28 us).  The weights are requested before anything waits: with
// BULK (independent calls on 4 MB or more) one thread bulk-copies the CTA's
// rows into shared memory (one copy per projection they fall in, completing
// on an mbarrier), so no register holds a load in flight and 5-6 calls' CTAs
// share an SM (4.4 MB calls: 1.62 -> 1.26 us against register-held loads);
// otherwise each lane loads its chunks into registers, all in flight at
// once.  The contraction is the same masked dp4a form; warp sums put row r,
// token m in lane r * MT + m, which dequantises and stores.  Everything but
// the output stores precedes griddepcontrol.wait for LAUNCH_PDL_INPUTS.
template <int MT, int R, int J, int NT, bool BULK>
__global__ void __launch_bounds__(NT) gemv_flat_kernel(LinearParams p) {
  // shared memory: (BULK) the CTA's weight rows (NT / 32 * R rows of ldw
  // bytes, as stored), then the activation codes as [MT][4][C] 16-byte units:
  // unit u of a token row (its inputs 16u .. 16u + 15) sits in plane u % 4 at
  // index u / 4, so the lanes of a warp, which hold consecutive chunks, read
  // consecutive 16-byte words
  extern __shared__ uint4 gs_smem[];
  __shared__ __align__(8) uint64_t s_wbar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = p.ldw / 16;                    // packed chunks per row
  // f / C = umulhi(f, ceil(2^32 / C)) exactly for f < 2^16 and 2 <= C <= 2^16
  // (the error term f (cmul C - 2^32) / 2^32 stays below 1 / C; C = 1 is f
  // itself): chunk f of the warp's rows is row f / C, chunk f % C of the
  // row, with no division and no dependence between chunks
  const uint32_t cmul = C > 1 ? 0xffffffffu / (uint32_t)C + 1u : 0u;
  constexpr int RB = (NT / 32) * R;            // weight rows of the CTA
  const int nb0 = blockIdx.x * RB;
  const int n0 = nb0 + warp * R;
  uint4* s_w = gs_smem;
  uint4* s_x = gs_smem + (BULK ? RB * C : 0);
  const bool inputs_ready = (p.flags & LAUNCH_PDL_INPUTS) != 0;
  const bool trigger_early = inputs_ready || (p.flags & LAUNCH_TRIGGER_EARLY) != 0;
  if (trigger_early) grid_launch_dependents();

  // 1. the weights, requested before anything waits.  BULK: the CTA's rows
  // by bulk copies (one per projection they fall in) completing on an
  // mbarrier; no register holds a load in flight, so several calls' CTAs fit
  // on an SM at once.  Otherwise every packed chunk of the warp's rows into
  // registers, all in flight at once (chunk f = lane + 32 j as row f / C,
  // chunk f % C of the row).
  uint4 w[BULK ? 1 : J];
  if constexpr (BULK) {
    if (threadIdx.x == 0) {
      mbar_init(&s_wbar, 1);
      fence_barrier_init();
      const int nb1 = nb0 + RB < p.N ? nb0 + RB : p.N;
      mbar_arrive_expect_tx(&s_wbar, (uint32_t)((nb1 - nb0) * p.ldw));
      for (int sg = 0; sg < p.nseg; ++sg) {
        const int lo = nb0 > p.seg_row0[sg] ? nb0 : p.seg_row0[sg];
        const int hi = nb1 < p.seg_row0[sg + 1] ? nb1 : p.seg_row0[sg + 1];
        if (lo < hi)
          bulk_load_1d(reinterpret_cast<uint8_t*>(s_w) + (size_t)(lo - nb0) * p.ldw,
                       p.seg_W[sg] + (size_t)(lo - p.seg_row0[sg]) * p.ldw,
                       (uint32_t)((hi - lo) * p.ldw), &s_wbar);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int f = lane + 32 * j;
      const int r = C > 1 ? (int)__umulhi((uint32_t)f, cmul) : f, c = f - r * C;
      w[j] = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);   // t = 0
      if (r < R && n0 + r < p.N) {
        int nl;
        const int sg = segment_of(p, n0 + r, nl);
        w[j] = ld_stream_v4(p.seg_W[sg] + (size_t)nl * p.ldw + 16 * c);
      }
    }
  }
  // the weight scale of this lane's output (lane r * MT + m: row n0 + r,
  // token m), part of the packed weights: fetched before any wait
  float gam = 0.0f;
  if (lane < R * MT && n0 + lane / MT < p.N) {
    int nl;
    gam = __ldg(p.seg_gamma[segment_of(p, n0 + lane / MT, nl)]);
  }

  // 2. activation codes, token scales and code sums
  if (!inputs_ready) {
    grid_dependency_wait();
    if (!trigger_early) grid_launch_dependents();
  }
  const int units = p.K / 16;
  for (int i = threadIdx.x; i < MT * units; i += NT) {
    const int m = i / units, u = i - m * units;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (m < p.M) v = *reinterpret_cast<const uint4*>(p.Xq + (size_t)m * p.K + 16 * u);
    s_x[(m * 4 + (u & 3)) * C + (u >> 2)] = v;
  }
  const int mt = lane < MT ? lane : 0;
  const bool tok = lane < p.M;
  const float s_m = tok ? p.xs[mt] : 1.0f;
  const int rs_m = tok ? p.xrs[mt] : 0;
  __syncthreads();                             // also publishes the barrier's initialisation
  if constexpr (BULK) {
    if (!mbar_wait(&s_wbar, 0u, nullptr)) {
      // never leave with a bulk copy in flight into this CTA's shared memory
      mbar_wait(&s_wbar, 0u, nullptr);
      return;
    }
  }

  // 3. unsigned codes x signed activations, per row and token.  Word u of a
  // chunk holds weight 16u + 4i + j at byte j, bits 2i; masking it with
  // 0x03030303 << 2i (no shift) leaves 4^i times the codes of weights
  // 16u + 4i .. 16u + 4i + 3, so the dp4a chain A_i of mask i carries a
  // factor 4^i, removed once per chunk: A_0 + A_1 / 4 + A_2 / 16 + A_3 / 64,
  // exact (each A_i is a multiple of 4^i; |A_i| < 2^19).
  int acc[R][MT];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0;
  // chunk f = lane + 32 j as (row r, chunk c of the row): with the weights
  // in registers (a dependent call, latency-bound) from f directly, so that
  // the chunks' shared-memory reads are independent; with bulk-copied
  // weights (independent calls, throughput-bound) stepped from the previous
  // chunk, which takes fewer instructions
  int r = 0, c = lane;
  if constexpr (BULK) {
    while (c >= C) {
      c -= C;
      ++r;
    }
  }
#pragma unroll
  for (int j = 0; j < J; ++j) {
    if constexpr (BULK) {
      if (j > 0) {
        c += 32;
        while (c >= C) {
          c -= C;
          ++r;
        }
      }
    } else {
      const int f = lane + 32 * j;
      r = C > 1 ? (int)__umulhi((uint32_t)f, cmul) : f;
      c = f - r * C;
    }
    if (r < R && n0 + r < p.N) {
      const uint4 wj = BULK ? s_w[(warp * R + r) * C + c] : w[j];
      const uint32_t wv[4] = {wj.x, wj.y, wj.z, wj.w};
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4* qp = s_x + m * 4 * C + c;           // 64 activation codes
        const uint4 qv[4] = {qp[0], qp[C], qp[2 * C], qp[3 * C]};
        int A[4] = {0, 0, 0, 0};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t q4[4] = {qv[u].x, qv[u].y, qv[u].z, qv[u].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) A[i] = dp4a_us(wv[u] & (0x03030303u << (2 * i)), q4[i], A[i]);
        }
        const int a = A[0] + (A[1] >> 2) + (A[2] >> 4) + (A[3] >> 6);
#pragma unroll
        for (int rr = 0; rr < R; ++rr)
          if (rr == r) acc[rr][m] += a;
      }
    }
  }

  // 4. warp sums; lane r * MT + m holds row r, token m, and forms its own
  // dequant factor (the row's projection sets gamma)
  float y = 0.0f;
  int yint = 0;
  int my_r = -1, my_m = 0;
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      int v = acc[r][m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      const int rs = __shfl_sync(0xffffffffu, rs_m, m);
      const float sm = __shfl_sync(0xffffffffu, s_m, m);
      if (lane == r * MT + m) {
        my_r = r;
        my_m = m;
        yint = v - rs;
        y = sm;                                  // the token's scale, for now
      }
    }
  const int n = n0 + my_r;
  int nl = 0, sg = 0;
  const bool valid = my_r >= 0 && my_m < p.M && n < p.N;
  if (valid) {
    sg = segment_of(p, n, nl);
    if (p.out_type != OUT_I32) {
      float fh, fl;
      dequant_factor(gam, y, fh, fl);
      y = dequant_dw(yint, fh, fl);
    }
  }
  if (inputs_ready) grid_dependency_wait();    // Y may still be read or written before
  if (valid) {
    const int Ns = p.seg_row0[sg + 1] - p.seg_row0[sg];
    const size_t idx = (size_t)my_m * Ns + nl;
    if (p.out_type == OUT_I32)
      reinterpret_cast<int32_t*>(p.seg_Y[sg])[idx] = yint;
    else
      store_value(p.seg_Y[sg], p.resid, idx, y, p.out_type, p.flags);
  }
}

}  // namespace bitnet
