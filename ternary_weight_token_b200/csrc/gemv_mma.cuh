// gemv_mma.cuh -- decode BitLinear (1..16 tokens) with short-lived CTAs:
// packed weight rows bulk-copied into shared memory, the contraction on
// warp-level int8 tensor-core instructions (mma.sync m16n8k32, u8 weight
// codes c = t + 1 x s8 activation codes, int32 accumulators).
//
// nnterp encyclopedia "bitnet", "The projections quantize their inputs and
// weights": the output equals the linear map of the rounded input by the
// ternarised weight exactly; the sum over k of q * c minus the token's sum of
// q is that exact int32 contraction.
//
// One CTA per 16 * RT weight rows (the rows of the call's projections,
// concatenated), every input of those rows:
//   - thread 0 issues one bulk copy per run of contiguous weight rows into
//     shared memory and, once the preceding grid has completed (or at once
//     when the caller states it writes none of the inputs), one for all the
//     activation rows (dense rows: the fragment loads of 8 rows share banks,
//     which costs less than the copy engine's time per extra copy);
//   - the 8 warps split the K steps of 32; each thread takes its A fragment
//     words straight from the packed rows (two 16-weight words per step, its
//     4-weight group picked by a shift and mask) and its B fragment words
//     from the activation rows; tokens past M read as zero;
//   - the warps add their int32 sums in shared memory (exact in any order);
//   - 64 threads per 16-row tile dequantise (gamma / s as an fp32 head and
//     tail, Sigma q subtracted) and store, after the dependency wait when the
//     loads went ahead of it.
// No cluster, no tensor memory, a few tens of KB of shared memory: CTAs are
// short-lived and several calls' CTAs share an SM.
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

constexpr int kGmThreads = 256;

struct GmParams {
  LinearParams lp;
  int rows_per_cta;            // 16 * RT
  int sw;                      // staged weight row stride (ldw + 16)
  int sx;                      // staged activation row stride (K + 16)
  int off_x;                   // activation rows after the weight rows
};

__device__ __forceinline__ void gm_mma(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void gm_bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int RT, int NTILE>
__global__ void __launch_bounds__(kGmThreads) gemv_mma_kernel(GmParams gp) {
  const LinearParams& p = gp.lp;
  extern __shared__ uint8_t gm_smem_raw[];
  __shared__ int red[RT * NTILE * 32 * 4];
  __shared__ __align__(8) uint64_t bar_w, bar_x;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(gm_smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* s_w = smem;                                   // [16 RT][sw]
  const int8_t* s_x = reinterpret_cast<const int8_t*>(smem + gp.off_x);   // [M][sx]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, c4 = lane & 3;
  const int row0 = blockIdx.x * (16 * RT);
  const int nrows = min(16 * RT, p.N - row0);
  const bool inputs_ready = (p.flags & LAUNCH_PDL_INPUTS) != 0;
  grid_launch_dependents();

  if (threadIdx.x == 0) {
    mbar_init(&bar_w, 1);
    mbar_init(&bar_x, 1);
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < RT * NTILE * 32 * 4; i += kGmThreads) red[i] = 0;
  __syncthreads();                                       // barriers initialised, red zeroed
  if (threadIdx.x == 0) {
    // one bulk copy per run of rows within one projection (a CTA's rows span
    // at most the end of one projection and the start of the next): the
    // preceding work does not write the weights (LAUNCH_PDL)
    mbar_arrive_expect_tx(&bar_w, (uint32_t)(nrows * p.ldw));
    for (int r = 0; r < nrows;) {
      int nl;
      const int sg = segment_of(p, row0 + r, nl);
      const int run = min(nrows - r, p.seg_row0[sg + 1] - (row0 + r));
      gm_bulk_g2s(s_w + (size_t)r * gp.sw, p.seg_W[sg] + (size_t)nl * p.ldw,
                  (uint32_t)(run * p.ldw), &bar_w);
      r += run;
    }
    if (!inputs_ready) grid_dependency_wait();
    mbar_arrive_expect_tx(&bar_x, (uint32_t)(p.M * p.K));
    gm_bulk_g2s(smem + gp.off_x, p.Xq, (uint32_t)(p.M * p.K), &bar_x);   // all M rows at once
  }

  // per-token scale and code sum, read while the copies are in flight
  if (!inputs_ready) grid_dependency_wait();
  const int mt = lane < 16 ? lane : 0;
  const bool tok = lane < p.M;
  const float s_m = tok ? __ldg(p.xs + mt) : 1.0f;
  const int rs_m = tok ? __ldg(p.xrs + mt) : 0;

  bool ok = mbar_wait(&bar_w, 0, nullptr);
  ok = mbar_wait(&bar_x, 0, nullptr) && ok;
  {
    const int steps = p.K / 32;
    const int s_lo = warp * steps / 8, s_hi = (warp + 1) * steps / 8;
    int acc[RT][NTILE][4];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
      for (int t = 0; t < NTILE; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][t][e] = 0;
    const int last = nrows > 0 ? nrows - 1 : 0;
    for (int s = s_lo; s < s_hi; ++s) {
      uint32_t bf[NTILE][2];
#pragma unroll
      for (int t = 0; t < NTILE; ++t) {
        const int m = 8 * t + g8;
        bf[t][0] = bf[t][1] = 0u;
        if (m < p.M) {
          const int8_t* xr = s_x + (size_t)m * gp.sx + 32 * s + 4 * c4;
          bf[t][0] = *reinterpret_cast<const uint32_t*>(xr);
          bf[t][1] = *reinterpret_cast<const uint32_t*>(xr + 16);
        }
      }
#pragma unroll
      for (int i = 0; i < RT; ++i) {
        if (16 * i < nrows) {
          const int r0 = min(16 * i + g8, last), r1 = min(16 * i + 8 + g8, last);
          const uint2 lo = *reinterpret_cast<const uint2*>(s_w + (size_t)r0 * gp.sw + 8 * s);
          const uint2 hi = *reinterpret_cast<const uint2*>(s_w + (size_t)r1 * gp.sw + 8 * s);
          const uint32_t a0 = (lo.x >> (2 * c4)) & 0x03030303u;
          const uint32_t a2 = (lo.y >> (2 * c4)) & 0x03030303u;
          const uint32_t a1 = (hi.x >> (2 * c4)) & 0x03030303u;
          const uint32_t a3 = (hi.y >> (2 * c4)) & 0x03030303u;
#pragma unroll
          for (int t = 0; t < NTILE; ++t) gm_mma(acc[i][t], a0, a1, a2, a3, bf[t][0], bf[t][1]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
      for (int t = 0; t < NTILE; ++t)
        if (16 * i < nrows)
#pragma unroll
          for (int e = 0; e < 4; ++e) atomicAdd(&red[((i * NTILE + t) * 32 + lane) * 4 + e], acc[i][t][e]);
  }
  __syncthreads();

  // epilogue: thread (row tile ti, token tile tt, lane ln) -> rows
  // 16 ti + g and 16 ti + 8 + g (g = ln / 4), tokens 8 tt + 2 (ln % 4) + {0, 1}
  const int idx = threadIdx.x;
  const int tiles = RT * NTILE * 32;
  const int i_t = idx >> 5, ln = idx & 31;
  const int ti = i_t / NTILE, tt = i_t % NTILE;
  // token scale / code sum of token m sit in lane m of every warp: gather
  // this thread's two tokens with full-warp shuffles before any divergence
  float s_tok[2];
  int rs_tok[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int m = (8 * tt + 2 * (ln & 3) + e) & 31;
    s_tok[e] = __shfl_sync(0xffffffffu, s_m, m);
    rs_tok[e] = __shfl_sync(0xffffffffu, rs_m, m);
  }
  float y[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  int yi[2][2] = {{0, 0}, {0, 0}};
  int nidx[2] = {-1, -1};
  if (idx < tiles && ok) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = 16 * ti + 8 * half + (ln >> 2);
      if (r >= nrows) continue;
      nidx[half] = row0 + r;
      int nl;
      const int sg = segment_of(p, row0 + r, nl);
      const float g = __ldg(p.seg_gamma[sg]);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int m = 8 * tt + 2 * (ln & 3) + e;
        if (m >= p.M) continue;
        const int v = red[idx * 4 + 2 * half + e] - rs_tok[e];
        yi[half][e] = v;
        if (p.out_type != OUT_I32) {
          float fh, fl;
          dequant_factor(g, s_tok[e], fh, fl);
          y[half][e] = dequant_dw(v, fh, fl);
        }
      }
    }
  }
  if (inputs_ready) grid_dependency_wait();            // Y may still be read or written before
  if (idx < tiles && ok) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if (nidx[half] < 0) continue;
      int nl;
      const int sg = segment_of(p, nidx[half], nl);
      const int Ns = p.seg_row0[sg + 1] - p.seg_row0[sg];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int m = 8 * tt + 2 * (ln & 3) + e;
        if (m >= p.M) continue;
        const size_t o = (size_t)m * Ns + nl;
        if (p.out_type == OUT_I32)
          reinterpret_cast<int32_t*>(p.seg_Y[sg])[o] = yi[half][e];
        else
          store_value(p.seg_Y[sg], p.resid, o, y[half][e], p.out_type, p.flags);
      }
    }
  }
}

}  // namespace bitnet
