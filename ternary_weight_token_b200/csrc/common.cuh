// common.cuh -- device-side helpers shared by the BitLinear kernels:
// the device error word, bounded mbarrier waits, TMA loads and the tcgen05
// (5th-generation tensor core / tensor memory) instructions, written as inline
// PTX for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bitnet {

// ---------------------------------------------------------------- errors
// Device error word: kernels OR a code into it when a bounded wait gives up.
// The host reads and clears it in bitnet_check_device_error().
enum : unsigned { DEV_ERR_TIMEOUT = 1u };

__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void record_device_error(unsigned code) {
  atomicOr(&g_device_error, code);
}

// Upper bound on any single wait inside a kernel.  Correct runs wait
// microseconds; the bound only turns a lost arrival into an error status
// instead of a hung GPU.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// -------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// One potentially blocking test of the phase: the thread sleeps until the
// phase completes or about kSuspendHintNs pass, so waiting warps do not spin
// for issue slots.
constexpr uint32_t kSuspendHintNs = 20000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return done != 0;
}

// Wait until the phase with the given parity has completed.  Gives up after
// `limit_ns` (recording DEV_ERR_TIMEOUT and raising *abort) or as soon as
// another role raised *abort.  Returns true when the phase completed.  The
// global timer is read only after 16 unsuccessful (sleeping) polls, so a wait
// that completes in the normal course never pays for it.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort_flag,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  unsigned long long t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (abort_flag != nullptr && *abort_flag) return false;
      const unsigned long long now = global_timer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > limit_ns) {
        record_device_error(DEV_ERR_TIMEOUT);
        if (abort_flag != nullptr) *abort_flag = 1;
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------- TMA
// 2-D tiled bulk tensor load global -> shared, completing on an mbarrier.
// No multicast: every CTA fetches its own tiles.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map,
                                            uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// 2-D tiled bulk tensor store shared -> global (bulk-group completion).  The
// box is clipped to the tensor bounds, so ragged edges are not written.
// Untiled bulk copy global -> shared, completing on an mbarrier: both
// addresses 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* src, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int x,
                                             int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N committed bulk groups still read their shared source.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every committed bulk group has completed (writes visible).
__device__ __forceinline__ void bulk_wait_group_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA) before a bulk copy reads them.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on `bar` when every tcgen05.mma this thread issued so far has
// completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[tmem] x B[smem]^T, kind::i8 (int32 accumulate).
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor for kind::i8: D int32, A unsigned 8-bit (the stored
// ternary codes t + 1), B signed 8-bit (activation codes), both K-major.
__host__ __device__ constexpr uint32_t make_idesc_i8(int M, int N) {
  return (2u << 4)                                  // D format: S32
         | (0u << 7)                                // A format: U8
         | (1u << 10)                               // B format: S8
         | (0u << 15) | (0u << 16)                  // A, B K-major
         | ((uint32_t)(N >> 3) << 17)               // N / 8
         | ((uint32_t)(M >> 4) << 24);              // M / 16
}

// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzled
// canonical layout (rows of 128 bytes, 8-row atoms of 1024 bytes).
__device__ __forceinline__ uint64_t make_sdesc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);     // start address
  d |= (uint64_t)1u << 16;                          // leading byte offset (unused, 16 B)
  d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset: 8 rows x 128 B
  d |= (uint64_t)1u << 46;                          // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                          // layout: SWIZZLE_128B
  return d;
}

// 32 lanes x 32 columns of 32-bit TMEM -> registers (one column per register).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// 16 lanes x 8 columns per repetition, 4 repetitions along the columns.
// Thread t receives, for repetition j, r[4j + 0, 1] = lane t/4, columns
// 8j + 2(t%4) + {0, 1} and r[4j + 2, 3] = lane 8 + t/4, the same columns (the
// fragment layout of an m16n8 accumulator, which stmatrix stores).
__device__ __forceinline__ void tmem_ld_16x256b_x4(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Four 8x8 matrices of 16-bit values, stored transposed: register i of thread
// t holds elements (t/4, 2(t%4) + {0, 1}) of matrix i, and thread 8i + r gives
// the shared-memory address of row r of the stored (transposed) matrix i.
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t addr, uint32_t r0, uint32_t r1,
                                                  uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(
                   addr),
               "r"(r0), "r"(r1), "r"(r2), "r"(r3)
               : "memory");
}

// Inverse of stmatrix_x4_trans: four 8x8 matrices of 16-bit values loaded
// transposed; thread 8i + r gives the address of row r of matrix i, and
// register i of thread t receives elements (t/4, 2(t%4) + {0, 1}) of matrix i.
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// registers -> 32 lanes x 32 columns of 32-bit TMEM.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Zero 32 lanes x 32 columns of TMEM (four 8-column stores of one zero
// register block, so no 32-register array stays live around the call).
__device__ __forceinline__ void tmem_zero_32x32b_x32(uint32_t taddr) {
  const uint32_t z = 0u;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
            taddr + 8u * k),
        "r"(z), "r"(z), "r"(z), "r"(z), "r"(z), "r"(z), "r"(z), "r"(z)
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Named barrier among `nthreads` threads (a multiple of 32) of the block.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------- grid-wide exchange
// For a cooperative launch (every CTA resident): each CTA publishes the
// launch's 64-bit epoch in its own flag once its global writes are done, and
// waits until every CTA's flag holds the epoch.  Epochs are never reused (the
// host draws a fresh one per launch from a counter started at a random
// value), so the flags need no reset and no zeroing.  Every thread of the CTA
// calls it; warp 0 polls (relaxed loads, then an acquire fence once every
// flag matched), bounded by kWaitLimitNs.  Returns false (device error
// recorded) if the wait gave up.
__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// `zero` / `nzero`: counters CTA 0 sets to 0 before it publishes its flag,
// so that no CTA can reach them (a later grid_count_exchange) before they
// are reset.
__device__ __forceinline__ bool grid_exchange(unsigned long long* flags, unsigned long long epoch,
                                              int* ok_smem, unsigned int* zero = nullptr,
                                              int nzero = 0) {
  __syncthreads();                               // this CTA's global writes are issued
  if (threadIdx.x == 0) {
    if (blockIdx.x == 0)
      for (int i = 0; i < nzero; ++i) zero[i] = 0u;
    __threadfence();
    st_release_u64(flags + blockIdx.x, epoch);
    *ok_smem = 1;
  }
  if (threadIdx.x < 32) {
    // every flag of a lane is loaded before any is compared (independent
    // relaxed loads in flight together), then one acquire fence
    const int lane = threadIdx.x;
    const unsigned long long t0 = global_timer_ns();
    bool done = false;
    for (uint32_t it = 0;; ++it) {
      int missing = 0;
      for (int i = lane; i < (int)gridDim.x; i += 32) missing += ld_relaxed_u64(flags + i) != epoch;
      done = __all_sync(0xffffffffu, missing == 0);
      if (done) break;
      if ((it & 7u) == 7u && global_timer_ns() - t0 > kWaitLimitNs) break;
    }
    if (!done && lane == 0) {
      record_device_error(DEV_ERR_TIMEOUT);
      *ok_smem = 0;
    }
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
  }
  __syncthreads();
  return *ok_smem != 0;
}

// Grid-wide exchange on an arrival counter that was reset to 0 within this
// launch (by a grid_exchange before it): thread 0 of each CTA makes the CTA's
// global writes visible (fence), adds 1, and polls the one counter word until
// all `expected` CTAs have arrived, bounded by kWaitLimitNs; then an acquire
// fence.  Polling one word costs about a third of polling every CTA's flag
// (measured on B200 with a 148-CTA cooperative grid: ~1.1 us against ~3 us
// per exchange).  Returns false (device error recorded) if the wait gave up.
__device__ __forceinline__ bool grid_count_exchange(unsigned int* ctr, unsigned int expected,
                                                    int* ok_smem) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
    const unsigned long long t0 = global_timer_ns();
    bool done = false;
    for (uint32_t it = 0;; ++it) {
      unsigned int v;
      asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
      if (v >= expected) {
        done = true;
        break;
      }
      if ((it & 15u) == 15u && global_timer_ns() - t0 > kWaitLimitNs) break;
    }
    if (!done) record_device_error(DEV_ERR_TIMEOUT);
    *ok_smem = done ? 1 : 0;
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
  }
  __syncthreads();
  return *ok_smem != 0;
}

// ------------------------------------------- programmatic dependent launch
// Wait until the grids this one depends on have completed and their memory
// is visible (returns at once for a launch without the PDL attribute).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Let the next grid on the stream start launching (its CTAs then wait in
// grid_dependency_wait until this grid has completed).
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// --------------------------------------------------------------- misc ALU
// SiLU y / (1 + e^-y) in fp32 ("bitnetv2-model" README, "Architecture
// Overview"): CUDA's expf (the full-precision function, not the fast
// intrinsic), an IEEE fp32 add, and the quotient as y times the hardware
// reciprocal (within 2 ulp; the IEEE division only for denominators beyond
// 2^126, where the reciprocal flushes to zero): a few fp32 ulp from the
// exact value.  One definition for every kernel that applies it, so the
// GEMM epilogue and the quantiser prelude give the same value.
__device__ __forceinline__ float silu_f32(float y) {
  const float d = __fadd_rn(1.0f, expf(-y));
  if (d < 0x1p126f) return __fdividef(y, d);
  return __fdiv_rn(y, d);
}

// Four unsigned bytes of `a` times four signed bytes of `b`, summed into c.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// 128-bit streaming load that bypasses L1 allocation (weights are read once).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Stored codes of 16 consecutive weights (one 32-bit word of the packed
// layout) -> four words, word j holding the codes of weights 4j..4j+3 one
// per byte.
__device__ __forceinline__ void expand_codes(uint32_t w, uint32_t& e0, uint32_t& e1,
                                             uint32_t& e2, uint32_t& e3) {
  e0 = w & 0x03030303u;
  e1 = (w >> 2) & 0x03030303u;
  e2 = (w >> 4) & 0x03030303u;
  e3 = (w >> 6) & 0x03030303u;
}

}  // namespace bitnet
