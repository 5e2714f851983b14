// gemv_tc.cuh -- decode BitLinear (M <= 16 tokens) on the tensor cores,
// split over K across a thread-block cluster.
//
// nnterp encyclopedia "bitnet", "The projections quantize their inputs and
// weights": the output equals the linear map of the rounded input by the
// ternarised weight exactly.  For a handful of tokens the projection is bound
// by streaming the packed weights (a quarter byte per weight) from HBM.
//
// Work split: the N weight rows are cut into 128-row tiles; each tile is
// handled by one cluster of S CTAs, CTA r taking a slice of the K inputs made
// of whole 64-input units (so every TMA coordinate stays 16-byte aligned), at
// most 7 chunks of 128.  Per CTA:
//   - one thread issues every TMA load of its slice at once (packed weights,
//     128 rows x 32 bytes per 128-k chunk; activation codes, 16 token rows x
//     128 bytes per chunk in the 128-byte swizzled layout), so the whole
//     slice is in flight;
//   - four converter warps expand each chunk's 2-bit codes to byte codes in
//     tensor memory (one TMEM lane per weight row) as soon as it lands, into
//     a ring of three 32-column slots; a slot is refilled once the
//     tcgen05.commit of the MMAs that read it has arrived;
//   - one thread issues tcgen05.mma kind::i8 (M = 128 weight rows, N = 16
//     tokens, K = 32) per 32-k step into a 16-column int32 accumulator;
//   - the four warps read the partial sums back (tcgen05.ld) and add those of
//     the valid tokens into one [16][128] buffer in the leader CTA's shared
//     memory (red.add over distributed shared memory), then arrive on the
//     leader's mbarrier with cluster-scope release;
//   - the leader waits (bounded) for all S arrivals, subtracts the token's
//     code sum, dequantises and writes the outputs.
// 128 TMEM columns and about 51 KB of shared memory per CTA: four CTAs
// (four consecutive calls) share an SM.
// With programmatic dependent launch the weight loads and their expansion
// start before the preceding kernel on the stream has finished; activation
// codes, scales and outputs are touched only after griddepcontrol.wait.  When
// the caller states that the preceding work writes none of the inputs
// (LAUNCH_PDL_INPUTS), everything up to the leader's output stores runs
// before that wait.
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

constexpr int kDecChunkK = 128;                 // k per TMA chunk
constexpr int kDecTokens = 16;                  // MMA N (tokens, zero-padded)
constexpr int kDecMaxChunks = 7;                // slice <= 896 inputs
constexpr int kDecMaxCluster = 8;
constexpr int kDecThreads = 192;                // warp 0 TMA+MMA, warp 1 alloc, warps 2-5 work
// D in columns [0, 16); converted weight chunks in a ring of three 32-column
// slots at columns 32, 64, 96 (a slot is refilled once the MMAs that read it
// have completed).  At most four CTAs share an SM (the shared-memory floor
// below), and 4 x 128 columns fit the 512 of an SM, so a CTA of a dependent
// launch can never hold the tensor memory its predecessor still needs.
constexpr int kDecTmemCols = 128;
constexpr int kDecASlots = 3;
constexpr int kDecMinSmem = 46 * 1024;          // at most four CTAs per SM

struct DecParams {
  int M, K;
  int units;              // K / 64
  const float* xs;
  const int32_t* xrs;
  const void* resid;
  int out_type;
  int flags;
  // projections sharing the activations: projection i owns the 128-row
  // tiles [seg_tile0[i], seg_tile0[i + 1]) and has seg_N[i] rows
  int nseg;
  int seg_tile0[kMaxSegments + 1];
  int seg_N[kMaxSegments];
  const float* seg_gamma[kMaxSegments];
  void* seg_Y[kMaxSegments];
};

// packed-weight tensor maps, one per projection
struct DecMaps {
  CUtensorMap w[kMaxSegments];
};

struct DecSmem {
  static constexpr int W_CHUNK = 128 * (kDecChunkK / 4);          // 4 KB
  static constexpr int X_CHUNK = kDecTokens * kDecChunkK;         // 2 KB
  static constexpr int OFF_X = 0;                                  // 1024-aligned chunks
  static constexpr int OFF_W = OFF_X + kDecMaxChunks * X_CHUNK;
  // leader: the cluster's partial sums, [16 tokens][128 rows] int32, which
  // every CTA of the cluster adds its own into (distributed shared memory)
  static constexpr int OFF_PART = OFF_W + kDecMaxChunks * W_CHUNK;
  static constexpr int PART_BYTES = kDecTokens * 128 * 4;          // 8 KB
  static constexpr int OFF_BAR = OFF_PART + PART_BYTES;
  // bars: wfull[chunks], xfull[chunks], afull[slots], aempty[slots], mma_done, reduce
  static constexpr int NUM_BARS = 2 * kDecMaxChunks + 2 * kDecASlots + 2;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024 > kDecMinSmem ? BYTES + 1024 : kDecMinSmem;
  static_assert(ALLOC <= 227 * 1024, "decode shared memory");
};

// Slice of the K inputs taken by cluster rank r: whole 64-input units, the
// first (units % S) ranks one unit more.
__device__ __forceinline__ void dec_slice(int units, int S, int r, int& k0, int& ks) {
  const int base = units / S, extra = units % S;
  k0 = 64 * (r * base + (r < extra ? r : extra));
  ks = 64 * (base + (r < extra ? 1 : 0));
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}

// Atomic add into a (possibly peer CTA's) shared-memory word of the cluster.
__device__ __forceinline__ void red_add_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_remote_release(uint32_t remote_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return done != 0;
}

// Bounded wait with cluster-scope acquire (partials written by peer CTAs).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
  unsigned long long t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 15u) == 0) {
      const unsigned long long now = global_timer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > limit_ns) {
        record_device_error(DEV_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// 32 lanes x 16 columns of 32-bit TMEM -> registers.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__global__ void __launch_bounds__(kDecThreads, 4)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                   const __grid_constant__ DecMaps maps, DecParams p) {
  extern __shared__ uint8_t dec_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dec_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sx = smem + DecSmem::OFF_X;
  uint8_t* sw = smem + DecSmem::OFF_W;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DecSmem::OFF_BAR);
  uint64_t* wfull = bars;                                 // [chunks] weight bytes landed
  uint64_t* xfull = bars + kDecMaxChunks;                 // [chunks] activation bytes landed
  uint64_t* afull = bars + 2 * kDecMaxChunks;             // [slots] a chunk's codes in TMEM
  uint64_t* aempty = afull + kDecASlots;                  // [slots] its MMAs completed
  uint64_t* mma_done = aempty + kDecASlots;               // accumulator complete
  uint64_t* reduce_bar = mma_done + 1;                    // leader: all partials in
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + DecSmem::OFF_MISC);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const int tile = blockIdx.x / (int)csize;               // 128-row weight tile
  int sg = 0;                                             // its projection
#pragma unroll
  for (int i = 1; i < kMaxSegments; ++i)
    if (i < p.nseg && tile >= p.seg_tile0[i]) sg = i;
  const int n0 = (tile - p.seg_tile0[sg]) * 128;          // first row within it
  const int Ns = p.seg_N[sg];
  const CUtensorMap* tm_w = &maps.w[sg];
  int k0, ks;
  dec_slice(p.units, (int)csize, (int)rank, k0, ks);
  const int chunks = (ks + kDecChunkK - 1) / kDecChunkK;
  // inputs not written by the preceding work: only the output stores wait
  const bool inputs_ready = (p.flags & LAUNCH_PDL_INPUTS) != 0;

  grid_launch_dependents();
  if (threadIdx.x == 0) {
    for (int c = 0; c < chunks; ++c) {
      mbar_init(&wfull[c], 1);
      mbar_init(&xfull[c], 1);
    }
    for (int a = 0; a < kDecASlots; ++a) {
      mbar_init(&afull[a], 4);                // four converter warps
      mbar_init(&aempty[a], 1);               // tcgen05.commit
    }
    mbar_init(mma_done, 1);
    mbar_init(reduce_bar, csize * 4);        // 4 storing warps per CTA
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kDecTmemCols);
    tmem_relinquish();
  }
  if (rank == 0) {                           // the partial sums start at zero
    uint32_t* part = reinterpret_cast<uint32_t*>(smem + DecSmem::OFF_PART);
    for (int i = threadIdx.x; i < kDecTokens * 128; i += kDecThreads) part[i] = 0u;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Arrive now, wait only before the first access to a peer's shared memory:
  // the leader's barrier initialisation then reaches every peer while they
  // stream their weights.
  cluster_arrive();
  const uint32_t tbase = *tmem_slot;
  const uint32_t a_col0 = 32;                // D occupies columns [0, 16)

  if (warp == 0) {
    if (lane == 0) {
      // weights do not depend on the preceding kernel: load them first
      tma_prefetch_desc(tm_w);
      for (int c = 0; c < chunks; ++c) {
        mbar_arrive_expect_tx(&wfull[c], DecSmem::W_CHUNK);
        tma_load_2d(sw + c * DecSmem::W_CHUNK, tm_w, &wfull[c], (k0 + c * kDecChunkK) / 4, n0);
      }
      if (!inputs_ready) grid_dependency_wait();   // activation codes from the previous kernel
      tma_prefetch_desc(&tm_x);
      for (int c = 0; c < chunks; ++c) {
        mbar_arrive_expect_tx(&xfull[c], DecSmem::X_CHUNK);
        tma_load_2d(sx + c * DecSmem::X_CHUNK, &tm_x, &xfull[c], k0 + c * kDecChunkK, 0);
      }
      // MMAs: 32-k steps of this CTA's slice
      const uint32_t idesc = make_idesc_i8(128, kDecTokens);
      const int steps = ks / 32;
      int s = 0;
      for (int c = 0; c < chunks; ++c) {
        const int slot = c % kDecASlots;
        if (!mbar_wait(&afull[slot], (uint32_t)(c / kDecASlots) & 1u, nullptr)) break;
        if (!mbar_wait(&xfull[c], 0, nullptr)) break;
        tc_fence_after();
        const uint32_t xaddr = smem_u32(sx + c * DecSmem::X_CHUNK);
        for (int j = 0; j < 4 && s < steps; ++j, ++s)
          mma_i8_ts(tbase, tbase + a_col0 + 32u * slot + 8u * j,
                    make_sdesc_sw128(xaddr + 32u * j), idesc, s > 0 ? 1u : 0u);
        tc_commit(&aempty[slot]);             // the slot is free once these complete
      }
      tc_commit(mma_done);
      // never leave bulk copies in flight
      for (int c = 0; c < chunks; ++c) {
        mbar_wait(&wfull[c], 0, nullptr, 100000000ull);
        mbar_wait(&xfull[c], 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
    cluster_wait();
  } else if (warp >= 2) {
    const int q = warp & 3;                  // TMEM lane quarter of this warp
    const int row = 32 * q + lane;           // weight row within the tile
    const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16);
    bool ok = true;
    for (int c = 0; c < chunks; ++c) {
      const int slot = c % kDecASlots;
      if (!mbar_wait(&wfull[c], 0, nullptr)) { ok = false; break; }
      if (c >= kDecASlots &&                  // the slot's previous chunk has been multiplied
          !mbar_wait(&aempty[slot], (uint32_t)(c / kDecASlots - 1) & 1u, nullptr)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint4* src = reinterpret_cast<const uint4*>(sw + c * DecSmem::W_CHUNK + row * 32);
      const uint4 a = src[0], b = src[1];
      uint32_t e[32];
      expand_codes(a.x, e[0], e[1], e[2], e[3]);
      expand_codes(a.y, e[4], e[5], e[6], e[7]);
      expand_codes(a.z, e[8], e[9], e[10], e[11]);
      expand_codes(a.w, e[12], e[13], e[14], e[15]);
      expand_codes(b.x, e[16], e[17], e[18], e[19]);
      expand_codes(b.y, e[20], e[21], e[22], e[23]);
      expand_codes(b.z, e[24], e[25], e[26], e[27]);
      expand_codes(b.w, e[28], e[29], e[30], e[31]);
      tmem_st_32x32b_x32(lane_base + a_col0 + 32u * slot, e);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[slot]);
    }
    // partial sums -> the leader's [token][row] sums (valid tokens only)
    uint32_t d[16];
    if (ok && mbar_wait(mma_done, 0, nullptr)) {
      tc_fence_after();
      tmem_ld_32x32b_x16(lane_base, d);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int t = 0; t < 16; ++t) d[t] = 0u;
    }
    cluster_wait();                          // the leader's barriers and zeroed sums exist
    const uint32_t part_remote =
        map_to_rank(smem_u32(smem + DecSmem::OFF_PART) + 4u * row, 0);
#pragma unroll
    for (int t = 0; t < 16; ++t)
      if (t < p.M) red_add_cluster_u32(part_remote + 4u * 128u * t, d[t]);
    __syncwarp();
    if (lane == 0) mbar_arrive_remote_release(map_to_rank(smem_u32(reduce_bar), 0));

    if (rank == 0) {
      // leader: token scales and code sums are fetched while the peers'
      // partials arrive; each token's dequant factor is formed once per warp
      // (lane m for token m, then shuffled); all partial sums are read and
      // every output value is computed before the first store, and with
      // LAUNCH_PDL_INPUTS before the wait for the preceding grid, so only
      // the stores follow it.
      if (!inputs_ready) grid_dependency_wait();
      const float g = __ldg(p.seg_gamma[sg]);
      const int mt = lane < kDecTokens ? lane : 0;
      const bool tok = lane < p.M;
      const float s_m = tok ? __ldg(p.xs + mt) : 1.0f;
      const int rs_m = tok ? __ldg(p.xrs + mt) : 0;
      float fh_m = 0.0f, fl_m = 0.0f;
      if (p.out_type != OUT_I32) dequant_factor(g, s_m, fh_m, fl_m);
      const bool all_in = mbar_wait_cluster(reduce_bar, 0);
      const int n = n0 + row;
      const int32_t* part = reinterpret_cast<const int32_t*>(smem + DecSmem::OFF_PART);
      int acc[kDecTokens];
#pragma unroll
      for (int m = 0; m < kDecTokens; ++m) acc[m] = -__shfl_sync(0xffffffffu, rs_m, m);
      if (all_in) {
#pragma unroll
        for (int m = 0; m < kDecTokens; ++m)
          if (m < p.M) acc[m] += part[m * 128 + row];
      }
      float y[kDecTokens];
#pragma unroll
      for (int m = 0; m < kDecTokens; ++m) {
        const float fh = __shfl_sync(0xffffffffu, fh_m, m);
        const float fl = __shfl_sync(0xffffffffu, fl_m, m);
        y[m] = p.out_type == OUT_I32 ? __int_as_float(acc[m]) : dequant_dw(acc[m], fh, fl);
      }
      if (inputs_ready) grid_dependency_wait();  // Y may still be read or written before
      if (all_in && n < Ns) {
#pragma unroll
        for (int m = 0; m < kDecTokens; ++m) {
          if (m < p.M) {
            const size_t idx = (size_t)m * Ns + n;
            if (p.out_type == OUT_I32)
              reinterpret_cast<int32_t*>(p.seg_Y[sg])[idx] = __float_as_int(y[m]);
            else
              store_value(p.seg_Y[sg], p.resid, idx, y[m], p.out_type, p.flags);
          }
        }
      }
    }
  } else {
    cluster_wait();                          // every thread of the cluster barrier waits once
  }

  // Peers only write into the leader's shared memory, and the leader leaves
  // only after all of them arrived, so no CTA of the cluster touches the
  // shared memory of a CTA that has exited.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kDecTmemCols);
}

}  // namespace bitnet
