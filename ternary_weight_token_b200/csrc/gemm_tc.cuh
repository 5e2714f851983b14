// gemm_tc.cuh -- prefill BitLinear on the sm_100a tensor cores
// (tcgen05.mma kind::i8, int32 accumulators in tensor memory).
//
// nnterp encyclopedia "bitnet", "The projections quantize their inputs and
// weights": the output equals the linear map of the rounded (int8) input by
// the ternarised weight exactly, dequantised by weight_scale / input scale.
// "The MLP gates with a squared ReLU" and "The block, in order" give the fused
// gate/up epilogue relu(g)^2 * u and the residual add; "bitnetv2-model"
// README, "Architecture Overview", the SiLU epilogue.
//
// Shape of the computation: D^T[n][m] = sum_k c[n][k] * q[m][k], where c = t + 1
// are the stored (unsigned) weight codes and q the signed activation codes;
// the epilogue subtracts sum_k q[m][k] to get the contraction with t.
//
//   A operand (M = 128 weight rows)  : tensor memory.  The packed 2-bit tile is
//       TMA-loaded into shared memory; converter warps expand each 32-bit word
//       of 16 codes into four words of byte codes (shift + mask) and write them
//       to tensor memory with tcgen05.st, one thread per row (TMEM lane).
//   B operand (N = BN tokens)        : shared memory, TMA-loaded int8 rows in the
//       128-byte swizzled K-major layout the MMA descriptor reads.
//   D (int32, 128 lanes x BN columns): tensor memory, double-buffered so the
//       epilogue of one tile overlaps the MMAs of the next.
//
// Warp roles (one persistent CTA per SM; 384 threads with one converter
// group, which keeps every role under the register cap with no spills):
//   warp 0        TMA producer (one thread)
//   warps 1, 3    MMA issuers (one thread each, alternate stages): 8 MMAs of
//                 K = 32 per 256-k stage, all accumulating into a buffer the
//                 epilogue zeroed
//   warp 2        tensor-memory allocator
//   warps 4..     converters (CONV_GROUPS groups of 4 warps alternate stages)
//   last 4 warps  epilogue: tcgen05.ld -> dequant -> fused op -> a 32 x 32
//                 tile staged in shared memory and written by a TMA store
//                 (plain stores when the output rows are not 16-byte multiples);
//                 bf16 outputs take the residual through a TMA load of the
//                 same 32 x 32 tile; GLU: each warp's TMEM quarter holds the
//                 gate rows and the up rows of the same 16 features (placed so
//                 by the converters), so m = relu(g)^2 * u forms in-thread
// Every wait is bounded; a wait that gives up records a device error, raises a
// CTA-wide abort flag, and the CTA drains its tensor-core work and bulk
// copies, frees tensor memory and exits.
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

template <int BN_, int BK_, int STAGES_, bool GLU_, bool SILU_ = false, int CONV_GROUPS_ = 1>
struct TcConfig {
  static constexpr int CONV_GROUPS = CONV_GROUPS_;  // converter warp groups (alternate stages)
  static constexpr bool SILU = SILU_;       // SiLU epilogue compiled in (H-BitLinear FFN)
  static constexpr int BN = BN_;            // tokens per tile (MMA N)
  static constexpr int BK = BK_;            // k per pipeline stage (multiple of 128)
  static constexpr int STAGES = STAGES_;
  // gate and up in one pass: the 128-row A tile stacks 64 gate rows over the
  // same 64 rows of the up weights, so a tile yields 64 output features
  static constexpr bool GLU = GLU_;
  static constexpr int BM = 128;            // weight rows per tile (MMA M, TMEM lanes)
  static constexpr int TILE_N = GLU ? BM / 2 : BM;   // output features per tile
  static constexpr int TOKF = GLU ? 2 : 1;  // dequant factors per token (gate, up)
  static constexpr int XSUB = BN * 128;     // one 128-byte-wide swizzled activation sub-tile
  static_assert(BK % 128 == 0 && BK <= 512, "BK");
  static constexpr int NW = 1;              // weight tiles per stage
  static constexpr int X_STAGE = BN * BK;   // bytes of activation codes per stage
  static constexpr int W_STAGE = BM * BK / 4;  // bytes of packed weights per matrix per stage
  static constexpr int ACC_COLS = BN * NW;  // TMEM columns per accumulator buffer
  static constexpr int A_COLS = (BK / 4) * NW;  // TMEM columns per A slot
  static constexpr int TMEM_COLS = 512;
  static_assert(2 * ACC_COLS + STAGES * A_COLS <= TMEM_COLS, "tensor memory overflow");
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
  static_assert(STAGES % CONV_GROUPS == 0, "converter groups alternate stages");
  static constexpr int EPI_WARP0 = 4 + 4 * CONV_GROUPS;
  static constexpr int THREADS = 32 * (EPI_WARP0 + 4);
  static constexpr int STAGE_OUT_BYTES = 32 * 32 * 4;          // one 32x32 output chunk (<= 4 B)
  static constexpr int OFF_X = 0;
  static constexpr int OFF_W = OFF_X + STAGES * X_STAGE;
  static constexpr int OFF_OUT = OFF_W + STAGES * NW * W_STAGE;  // 4 warps x 2 buffers
  static constexpr int OFF_BAR = OFF_OUT + 4 * 2 * STAGE_OUT_BYTES;
  static constexpr int NUM_BARS = 3 * STAGES + 7 + 8;    // + residual chunks (4 warps x 2)
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;   // slack for 1024-B alignment
  static constexpr uint32_t TX_BYTES = X_STAGE + NW * W_STAGE;
};

struct TcParams {
  int M, N, K;
  int num_kb;                 // k stages = ceil(K / BK)
  int tiles_n, num_tiles;
  const float* xs;            // [M] activation scales
  const int32_t* xrs;         // [M] sum of activation codes
  const float* gamma0;        // weight scale (gate weights for GLU)
  const float* gamma1;        // up weight scale (GLU only)
  void* Y;                    // [M][N]
  const void* resid;          // [M][N] or null
  int out_type;
  int flags;
  int tma_out;                // 1: output written through the TMA map tm_y
  int tma_res;                // 1: bf16 residual read through the TMA map tm_r
  int w_early;                // 1: the preceding work does not write the packed weights:
                              // the first stages' weight tiles load before the dependency wait
};

__device__ __forceinline__ int out_elem_bytes(int out_type) { return out_type == OUT_BF16 ? 2 : 4; }

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                   const __grid_constant__ CUtensorMap tm_w0,
                   const __grid_constant__ CUtensorMap tm_w1,
                   const __grid_constant__ CUtensorMap tm_y,
                   const __grid_constant__ CUtensorMap tm_r, TcParams p) {
  extern __shared__ uint8_t tc_smem_raw[];
  // per-token dequant factors (fp32 head, tail) and code sums of a tile,
  // computed once by the four epilogue warps; two buffers alternate between
  // consecutive tiles.  Static so they never alias the output staging buffers.
  __shared__ __align__(16) float2 s_tok_f[2][C::TOKF * C::BN];
  __shared__ __align__(16) int s_tok_rs[2][C::BN];

  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sx = smem + C::OFF_X;
  uint8_t* sw = smem + C::OFF_W;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                       // TMA bytes landed       (count 1 + tx)
  uint64_t* empty = bars + C::STAGES;          // MMAs done with stage   (tcgen05.commit)
  uint64_t* afull = bars + 2 * C::STAGES;      // A codes in TMEM        (4 converter warps)
  uint64_t* accfull = bars + 3 * C::STAGES;    // accumulator ready      (tcgen05.commit)
  uint64_t* accempty = accfull + 2;            // accumulator drained    (4 epilogue warps)
  uint64_t* drain = accempty + 2;              // teardown drain
  uint64_t* tokbar = drain + 1;                // tile's token factors written (4 warps)
  uint64_t* rbar = tokbar + 2;                 // [warp q][buffer] residual chunk landed (TMA)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&afull[s], 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 2);             // one commit from each MMA issuer
      mbar_init(&accempty[b], 4);            // four epilogue warps (zeroed buffer)
    }
    mbar_init(drain, 2);
    mbar_init(&tokbar[0], 4);
    mbar_init(&tokbar[1], 4);
    for (int b = 0; b < 8; ++b) mbar_init(&rbar[b], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w0);
    if (C::GLU) tma_prefetch_desc(&tm_w1);
    if (p.tma_out) tma_prefetch_desc(&tm_y);
    if (p.tma_res) tma_prefetch_desc(&tm_r);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Launched with programmatic dependent launch: the setup above touches no
  // global memory; everything below runs after the preceding grid completed,
  // except (w_early) the producer's loads of the first stages' weight tiles.
  grid_launch_dependents();
  if (!(p.w_early && warp == 0)) grid_dependency_wait();
  const uint32_t tbase = *tmem_slot;
  const uint32_t a_col0 = 2 * C::ACC_COLS;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      // w_early: the first tile's first stages (fresh barriers: no empty wait)
      // get their weight tiles before the dependency wait and their
      // activation tiles after it
      int pre = 0;
      if (p.w_early && (int)blockIdx.x < p.num_tiles) {
        const int tn = (int)blockIdx.x % p.tiles_n, tm = (int)blockIdx.x / p.tiles_n;
        pre = p.num_kb < C::STAGES ? p.num_kb : C::STAGES;
        for (int kb = 0; kb < pre; ++kb) {
          mbar_arrive_expect_tx(&full[kb], C::TX_BYTES);
          if (C::GLU) {
            tma_load_2d(sw + kb * C::W_STAGE, &tm_w0, &full[kb], kb * (C::BK / 4), tn * C::TILE_N);
            tma_load_2d(sw + kb * C::W_STAGE + (C::BM / 2) * (C::BK / 4), &tm_w1, &full[kb],
                        kb * (C::BK / 4), tn * C::TILE_N);
          } else {
            tma_load_2d(sw + kb * C::W_STAGE, &tm_w0, &full[kb], kb * (C::BK / 4), tn * C::BM);
          }
        }
        grid_dependency_wait();
        for (int kb = 0; kb < pre; ++kb) {
#pragma unroll
          for (int xs = 0; xs < C::BK / 128; ++xs)
            tma_load_2d(sx + kb * C::X_STAGE + xs * C::XSUB, &tm_x, &full[kb],
                        kb * C::BK + 128 * xs, tm * C::BN);
        }
        it = (uint32_t)pre;
      } else if (p.w_early) {
        grid_dependency_wait();
      }
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        const int tn = tile % p.tiles_n, tm = tile / p.tiles_n;
        for (int kb = tile == (int)blockIdx.x ? pre : 0; kb < p.num_kb; ++kb, ++it) {
          const uint32_t st = it % C::STAGES, ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) goto producer_done;
          mbar_arrive_expect_tx(&full[st], C::TX_BYTES);
#pragma unroll
          for (int xs = 0; xs < C::BK / 128; ++xs)
            tma_load_2d(sx + st * C::X_STAGE + xs * C::XSUB, &tm_x, &full[st],
                        kb * C::BK + 128 * xs, tm * C::BN);
          if (C::GLU) {                       // rows 0-63 gate, 64-127 up
            tma_load_2d(sw + st * C::W_STAGE, &tm_w0, &full[st], kb * (C::BK / 4),
                        tn * C::TILE_N);
            tma_load_2d(sw + st * C::W_STAGE + (C::BM / 2) * (C::BK / 4), &tm_w1, &full[st],
                        kb * (C::BK / 4), tn * C::TILE_N);
          } else {
            tma_load_2d(sw + st * C::W_STAGE, &tm_w0, &full[st], kb * (C::BK / 4), tn * C::BM);
          }
        }
      }
    producer_done:
      // Never leave bulk copies in flight: wait for the last issued stages.
      const uint32_t last = it < (uint32_t)C::STAGES ? it : (uint32_t)C::STAGES;
      for (uint32_t i = 0; i < last; ++i) {
        const uint32_t j = it - 1 - i;
        mbar_wait(&full[j % C::STAGES], (j / C::STAGES) & 1u, nullptr, 100000000ull);
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------ MMA issuers
    // Two threads issue the MMAs of alternate stages, so one waits for its
    // next stage while the tensor pipe runs the other's.  Every MMA
    // accumulates (int32 sums are exact in any order); the epilogue zeroes an
    // accumulator buffer after reading it, before handing it back.
    if (lane == 0) {
      const uint32_t me = warp == 1 ? 0u : 1u;
      const uint32_t idesc = make_idesc_i8(C::BM, C::BN);
      uint32_t it = 0, tcount = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
        const uint32_t ab = tcount & 1u, use = tcount >> 1;
        if (!mbar_wait(&accempty[ab], use & 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_col = tbase + ab * C::ACC_COLS;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          if ((it & 1u) != me) continue;
          const uint32_t st = it % C::STAGES, ph = (it / C::STAGES) & 1u;
          // The converters arrive on afull[st] only after they observed full[st]
          // complete, so this one wait also orders the MMA after the TMA bytes.
          if (!mbar_wait(&afull[st], ph, abort_flag)) goto mma_done;
          tc_fence_after();
          const uint32_t a_col = tbase + a_col0 + st * C::A_COLS;
          const uint32_t xaddr = smem_u32(sx + st * C::X_STAGE);
#pragma unroll
          for (int j = 0; j < C::BK / 32; ++j) {
            const uint64_t bdesc =
                make_sdesc_sw128(xaddr + (uint32_t)((j >> 2) * C::XSUB) + 32u * (j & 3));
            mma_i8_ts(d_col, a_col + 8u * j, bdesc, idesc, 1u);
          }
          tc_commit(&empty[st]);
        }
        tc_commit(&accfull[ab]);
      }
    mma_done:
      tc_commit(drain);
      mbar_wait(drain, 0, nullptr, 100000000ull);
    }
  } else if (warp >= 4 && warp < C::EPI_WARP0) {
    // ------------------------------------------------------- converters
    const uint32_t group = (uint32_t)(warp - 4) >> 2;   // stages with it % groups == group
    const int q = warp & 3;
    // TMEM lane 32 q + lane holds weight row `row` of the stage: the row
    // itself, or for GLU the gate row 16 q + lane (lane < 16) and the up row
    // 64 + 16 q + lane - 16, so each epilogue warp's quarter holds the gate
    // and up rows of the same 16 features
    const int row = C::GLU ? (lane < 16 ? 16 * q + lane : 48 + 16 * q + lane) : 32 * q + lane;
    const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16) + a_col0;
    const uint32_t total = (uint32_t)((p.num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) /
                                      (int)gridDim.x) * (uint32_t)p.num_kb;
    for (uint32_t it = group; it < total; it += C::CONV_GROUPS) {
      const uint32_t st = it % C::STAGES, ph = (it / C::STAGES) & 1u;
      if (!mbar_wait(&full[st], ph, abort_flag)) break;
      tc_fence_after();
#pragma unroll
      for (int w = 0; w < C::NW; ++w) {
        // Packed rows are BK/4 bytes; TMA wrote them with the matching swizzle
        // (16-byte chunk j of row r at chunk j ^ ((r / (128 / row_bytes)) %
        // chunks)), so the 32 lanes' 16-byte loads hit distinct banks.
        const uint4* src = reinterpret_cast<const uint4*>(sw + (st * C::NW + w) * C::W_STAGE +
                                                          row * (C::BK / 4));
        constexpr int CH = C::BK / 64;            // 16-byte chunks per packed row (2 or 4)
        const int swz = (row / (8 / CH)) & (CH - 1);
#pragma unroll
        for (int h = 0; h < C::BK / 128; ++h) {   // 128 weights -> 32 TMEM columns
          const uint4 a = src[(2 * h) ^ swz], b = src[(2 * h + 1) ^ swz];
          uint32_t e[32];
          expand_codes(a.x, e[0], e[1], e[2], e[3]);
          expand_codes(a.y, e[4], e[5], e[6], e[7]);
          expand_codes(a.z, e[8], e[9], e[10], e[11]);
          expand_codes(a.w, e[12], e[13], e[14], e[15]);
          expand_codes(b.x, e[16], e[17], e[18], e[19]);
          expand_codes(b.y, e[20], e[21], e[22], e[23]);
          expand_codes(b.z, e[24], e[25], e[26], e[27]);
          expand_codes(b.w, e[28], e[29], e[30], e[31]);
          tmem_st_32x32b_x32(lane_base + st * C::A_COLS + (C::BK / 4) * w + 32u * h, e);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[st]);
    }
  } else if (warp >= C::EPI_WARP0) {
    // --------------------------------------------------------- epilogue
    const int q = warp & 3;
    const float g0 = __ldg(p.gamma0);
    const float g1 = C::GLU ? __ldg(p.gamma1) : 0.0f;
    const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16);
    const int esz = out_elem_bytes(p.out_type);
    const uint32_t out_base = smem_u32(smem + C::OFF_OUT + q * 2 * C::STAGE_OUT_BYTES);
    // bf16 output through the TMA store: fragment epilogue (16x256b loads,
    // transposing stmatrix into a 64-byte-swizzled staging tile)
    const bool frag_path = !C::GLU && p.tma_out && p.out_type == OUT_BF16;
    // both accumulator buffers start at zero: every MMA accumulates
    for (int col = 0; col < 2 * C::ACC_COLS; col += 32) tmem_zero_32x32b_x32(lane_base + col);
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&accempty[0]);
      mbar_arrive(&accempty[1]);
    }
    uint32_t tcount = 0, chunk_count = 0;
    uint32_t rphase = 0;                         // bit b: parity of this warp's rbar[b]
    // bf16 residual of a 32 x 32 output chunk: one TMA load into the upper
    // half of the chunk's staging buffer (64-byte swizzled like the output
    // staging), issued a chunk ahead, read back with ldmatrix.trans
    const bool res_tma = frag_path && p.tma_res && (p.flags & EPI_RESIDUAL);
    auto res_load = [&](uint32_t cc, int nq, int mrow) {
      const uint32_t b = cc & 1u;
      const uint32_t dst = out_base + b * C::STAGE_OUT_BYTES + 2048u;
      if (lane == 0) {
        mbar_arrive_expect_tx(&rbar[2 * q + b], 2048u);
        tma_load_2d(smem + (dst - smem_u32(smem)), &tm_r, &rbar[2 * q + b], nq, mrow);
      }
    };
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
      const int tn = tile % p.tiles_n, tm = tile / p.tiles_n;
      const int m0 = tm * C::BN;
      // first output feature of this warp (GLU: warps 0-1 hold gate rows,
      // warps 2-3 the up rows of the same features)
      const int nq0 = tn * C::TILE_N + 32 * (C::GLU ? (q & 1) : q);
      if (res_tma && nq0 < p.N && m0 < p.M) res_load(chunk_count, nq0, m0);
      const uint32_t ab = tcount & 1u, aph = (tcount >> 1) & 1u;
      float2* tok_f = s_tok_f[ab];               // [NW][BN]
      int* tok_rs = s_tok_rs[ab];
      // This buffer was last read for tile tcount - 2; every warp has since
      // arrived on the other buffer's barrier, so no warp still reads it.
      for (int j = 32 * q + lane; j < C::BN; j += 128) {
        const int m = m0 + j;
        float2 f0 = make_float2(0.0f, 0.0f), f1 = make_float2(0.0f, 0.0f);
        int rs = 0;
        if (m < p.M) {
          const float s = p.xs[m];
          dequant_factor(g0, s, f0.x, f0.y);
          if (C::GLU) dequant_factor(g1, s, f1.x, f1.y);
          rs = p.xrs[m];
        }
        tok_f[j] = f0;
        if (C::GLU) tok_f[C::BN + j] = f1;
        tok_rs[j] = rs;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&tokbar[ab]);
      if (!mbar_wait(&tokbar[ab], aph, abort_flag)) break;
      if (!mbar_wait(&accfull[ab], aph, abort_flag)) break;
      tc_fence_after();
      const int n = nq0 + lane;
      const bool n_ok = n < p.N;
#pragma unroll 1
      for (int c = 0; c < C::BN / 32; ++c, ++chunk_count) {
        const int mc = m0 + 32 * c;              // first token of this chunk
        if (mc >= p.M) {                         // past the last token: only re-zero
          tmem_zero_32x32b_x32(lane_base + ab * C::ACC_COLS + 32u * c);
          continue;
        }
        if constexpr (!C::GLU) {
          if (frag_path) {
            // v[16h + 4j + k]: weight row nq0 + 16h + 8(k / 2) + lane / 4,
            // token mc + 8j + 2(lane % 4) + k % 2
            uint32_t v[32];
            tmem_ld_16x256b_x4(lane_base + ab * C::ACC_COLS + 32u * c, v);
            tmem_ld_16x256b_x4(lane_base + (16u << 16) + ab * C::ACC_COLS + 32u * c, v + 16);
            const int tq = 2 * (lane & 3);       // this thread's even token offset
            // the next chunk's residual goes in flight before this one is used
            if (res_tma && c + 1 < C::BN / 32 && mc + 32 < p.M && nq0 < p.N)
              res_load(chunk_count + 1, nq0, mc + 32);
            // residual (bf16) of the same elements, two per register
            uint32_t rpk[16];
            if ((p.flags & EPI_RESIDUAL) && !res_tma) {
              const uint16_t* rp = reinterpret_cast<const uint16_t*>(p.resid);
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                const int nn = nq0 + 16 * (i >> 4) + 8 * ((i >> 1) & 1) + (lane >> 2);
                const int mm = mc + 8 * ((i >> 2) & 3) + tq;
                const bool ok = nn < p.N;
                const uint32_t lo = (ok && mm < p.M) ? rp[(size_t)mm * p.N + nn] : 0u;
                const uint32_t hi = (ok && mm + 1 < p.M) ? rp[(size_t)(mm + 1) * p.N + nn] : 0u;
                rpk[i >> 1] = lo | (hi << 16);
              }
            }
            tmem_ld_wait();
            tmem_zero_32x32b_x32(lane_base + ab * C::ACC_COLS + 32u * c);
            // staging tile: 32 token rows of 64 bytes (32 weight rows, bf16),
            // 16-byte chunk k of row m at chunk k ^ ((m / 2) % 4) (64-byte swizzle)
            const uint32_t buf = out_base + (chunk_count & 1u) * C::STAGE_OUT_BYTES;
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
            const int mi = lane >> 3, rr8 = lane & 7;
            if (res_tma && nq0 < p.N) {
              const uint32_t b = chunk_count & 1u;
              if (!mbar_wait(&rbar[2 * q + b], (rphase >> b) & 1u, abort_flag)) break;
              rphase ^= 1u << b;
              const uint32_t rb = buf + 2048u;
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int jp = 0; jp < 2; ++jp) {
                  const int row = 8 * (2 * jp + (mi >> 1)) + rr8;
                  const int chunk = (2 * h + (mi & 1)) ^ ((row >> 1) & 3);
                  ldmatrix_x4_trans(rb + (uint32_t)(row * 64 + chunk * 16), rpk[8 * h + 4 * jp + 0],
                                    rpk[8 * h + 4 * jp + 1], rpk[8 * h + 4 * jp + 2],
                                    rpk[8 * h + 4 * jp + 3]);
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {        // weight rows nq0 + 16h .. + 15
              uint32_t pk[8];                    // bf16x2 of matrix (j, s): pk[2j + s]
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int t = 32 * c + 8 * j + tq;
                const float4 ff = *reinterpret_cast<const float4*>(&tok_f[t]);
                const int2 rr = *reinterpret_cast<const int2*>(&tok_rs[t]);
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2) {
                  const int i = 16 * h + 4 * j + 2 * s2;
                  float y0 = dequant_dw((int)v[i] - rr.x, ff.x, ff.y);
                  float y1 = dequant_dw((int)v[i + 1] - rr.y, ff.z, ff.w);
                  if (C::SILU) {
                    y0 = silu_f32(y0);
                    y1 = silu_f32(y1);
                  }
                  if (p.flags & EPI_RESIDUAL) {
                    // TMA path: residual pair of matrix (j, s2) of half h
                    const uint32_t rr2 = res_tma ? rpk[8 * h + 2 * j + s2] : rpk[i >> 1];
                    y0 = __fadd_rn(__uint_as_float(rr2 << 16), y0);
                    y1 = __fadd_rn(__uint_as_float(rr2 & 0xffff0000u), y1);
                  }
                  const __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
                  pk[2 * j + s2] = *reinterpret_cast<const uint32_t*>(&b2);
                }
              }
#pragma unroll
              for (int jp = 0; jp < 2; ++jp) {
                // matrix mi of this store: token block j = 2 jp + mi / 2,
                // weight-row block 8 (mi % 2) of half h
                const int row = 8 * (2 * jp + (mi >> 1)) + rr8;
                const int chunk = (2 * h + (mi & 1)) ^ ((row >> 1) & 3);
                stmatrix_x4_trans(buf + (uint32_t)(row * 64 + chunk * 16), pk[4 * jp + 0],
                                  pk[4 * jp + 1], pk[4 * jp + 2], pk[4 * jp + 3]);
              }
            }
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0 && nq0 < p.N) {
              tma_store_2d(&tm_y, smem + (buf - smem_u32(smem)), nq0, mc);
              bulk_commit_group();
            }
            continue;
          }
        }
        if constexpr (C::GLU) {
          // lanes 32 q .. + 15 hold gate rows, 32 q + 16 .. + 31 the up rows
          // of the same 16 features: v[4j + k] (gate) and v[16 + 4j + k] (up)
          // are feature fq0 + 8 (k / 2) + lane / 4, token mc + 8 j +
          // 2 (lane % 4) + k % 2, so m = relu(g)^2 * u forms in the thread
          uint32_t v[32];
          tmem_ld_16x256b_x4(lane_base + ab * C::ACC_COLS + 32u * c, v);
          tmem_ld_16x256b_x4(lane_base + (16u << 16) + ab * C::ACC_COLS + 32u * c, v + 16);
          tmem_ld_wait();
          tmem_zero_32x32b_x32(lane_base + ab * C::ACC_COLS + 32u * c);
          const int tq = 2 * (lane & 3);
          const int fq0 = tn * C::TILE_N + 16 * q;   // first feature of this warp
          float mv[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int t = 32 * c + 8 * j + tq;
            const float4 fg = *reinterpret_cast<const float4*>(&tok_f[t]);
            const float4 fu = *reinterpret_cast<const float4*>(&tok_f[C::BN + t]);
            const int2 rr = *reinterpret_cast<const int2*>(&tok_rs[t]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int i = 4 * j + k;
              const bool odd = (k & 1) != 0;
              const int rs = odd ? rr.y : rr.x;
              const float g = dequant_dw((int)v[i] - rs, odd ? fg.z : fg.x, odd ? fg.w : fg.y);
              const float u = dequant_dw((int)v[16 + i] - rs, odd ? fu.z : fu.x, odd ? fu.w : fu.y);
              mv[i] = __fmul_rn(g > 0.0f ? __fmul_rn(g, g) : 0.0f, u);
            }
          }
          if (p.tma_out) {
            // 32 tokens x 16 features fp32 staged as 64-byte token rows
            const uint32_t buf = out_base + (chunk_count & 1u) * C::STAGE_OUT_BYTES;
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int trel = 8 * (i >> 2) + tq + (i & 1);
              const int frel = 8 * ((i >> 1) & 1) + (lane >> 2);
              st_shared_u32(buf + (uint32_t)(trel * 64 + frel * 4), __float_as_uint(mv[i]));
            }
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0 && fq0 < p.N) {
              tma_store_2d(&tm_y, smem + (buf - smem_u32(smem)), fq0, mc);
              bulk_commit_group();
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int m = mc + 8 * (i >> 2) + tq + (i & 1);
              const int n = fq0 + 8 * ((i >> 1) & 1) + (lane >> 2);
              if (m < p.M && n < p.N) reinterpret_cast<float*>(p.Y)[(size_t)m * p.N + n] = mv[i];
            }
          }
          continue;
        }
        uint32_t v[32];
        float y[32];
        tmem_ld_32x32b_x32(lane_base + ab * C::ACC_COLS + 32u * c, v);
        {
          tmem_ld_wait();
          tmem_zero_32x32b_x32(lane_base + ab * C::ACC_COLS + 32u * c);
          if (p.out_type == OUT_I32) {
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = __int_as_float((int)v[j] - tok_rs[32 * c + j]);
          } else {
            // residual of this chunk: 32 independent loads issued back to back
            // (one dtype branch for the whole chunk), before the dequant math
            float r[32];
            if (!C::SILU && (p.flags & EPI_RESIDUAL)) {
              if (p.out_type == OUT_BF16) {
                const __nv_bfloat16* rp = reinterpret_cast<const __nv_bfloat16*>(p.resid);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  r[j] = (n_ok && mc + j < p.M) ? __bfloat162float(rp[(size_t)(mc + j) * p.N + n])
                                                : 0.0f;
              } else {
                const float* rp = reinterpret_cast<const float*>(p.resid);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  r[j] = (n_ok && mc + j < p.M) ? rp[(size_t)(mc + j) * p.N + n] : 0.0f;
              }
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int t = 32 * c + j;
              const float2 fa = tok_f[t];
              float yy = dequant_dw((int)v[j] - tok_rs[t], fa.x, fa.y);
              if (C::SILU) yy = silu_f32(yy);   // only the SiLU instance carries expf
              if (p.flags & EPI_RESIDUAL) {
                if (C::SILU) {          // rare combination: plain per-element load
                  const int m = mc + j;
                  if (n_ok && m < p.M) {
                    const size_t idx = (size_t)m * p.N + n;
                    yy = __fadd_rn(p.out_type == OUT_BF16
                                       ? __bfloat162float(
                                             reinterpret_cast<const __nv_bfloat16*>(p.resid)[idx])
                                       : reinterpret_cast<const float*>(p.resid)[idx],
                                   yy);
                  }
                } else {
                  yy = __fadd_rn(r[j], yy);
                }
              }
              y[j] = yy;
            }
          }
        }
        if (p.tma_out) {
          // stage the 32 (tokens) x 32 (weight rows) chunk as rows of the
          // output, then one TMA store; two buffers per warp alternate
          const uint32_t buf = out_base + (chunk_count & 1u) * C::STAGE_OUT_BYTES;
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          if (esz == 2) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              st_shared_u16(buf + (uint32_t)(j * 32 + lane) * 2u,
                            __bfloat16_as_ushort(__float2bfloat16_rn(y[j])));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              st_shared_u32(buf + (uint32_t)(j * 32 + lane) * 4u, __float_as_uint(y[j]));
          }
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0 && nq0 < p.N) {
            tma_store_2d(&tm_y, smem + (buf - smem_u32(smem)), nq0, mc);
            bulk_commit_group();
          }
        } else if (n_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = mc + j;
            if (m < p.M) {
              const size_t idx = (size_t)m * p.N + n;
              if (p.out_type == OUT_BF16)
                reinterpret_cast<__nv_bfloat16*>(p.Y)[idx] = __float2bfloat16_rn(y[j]);
              else
                reinterpret_cast<float*>(p.Y)[idx] = y[j];   // fp32, or int32 bits
            }
          }
        }
      }
      tmem_st_wait();                            // the zeroed buffer is complete
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[ab]);
    }
    if (lane == 0) bulk_wait_group_all();      // output stores complete before exit
    __syncwarp();
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tbase, C::TMEM_COLS);
}

}  // namespace bitnet
