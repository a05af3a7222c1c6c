// Block-scaled NVFP4 GEMM on the sm_100a 5th-generation tensor cores.
//
//   out[m, n] = epi(alpha_a * alpha_b * sum_k a_mk * sA[m, k/16] * b_nk * sB[n, k/16])
//
// A [M, K] and B [N, K] are packed E2M1 codes (K-major), sA / sB are UE4M3
// scales in the tcgen05 block-scaled layout.  Persistent kernel of CTA pairs
// (clusters of two on neighbouring SMs): each pair walks 256 x 256 output
// tiles in a grouped (L2-friendly) order with 2-SM MMAs
// (tcgen05.mma.cta_group::2, M = 256): CTA r of the pair holds A rows
// [128 r, 128 r + 128) and B rows [128 r, 128 r + 128) of the tile in shared
// memory and output rows [128 r, 128 r + 128) in tensor memory, so each SM
// stores and serves only half of B -- the operand traffic through shared
// memory per MMA is two thirds of a single-SM 128 x 256 tile's.
//   warp 0       TMA producer (both CTAs): each CTA loads its own code tiles
//                with the 2-SM form of cp.async.bulk.tensor (completion
//                counted on the leader CTA's barrier) and its scale atoms
//                with cp.async.bulk, a 5-deep ring that runs ahead across
//                tiles;
//   warp 1       allocates tensor memory (cta_group::2); in the leader CTA one
//                thread issues the four MMAs (kind::mxf4nvf4, block16 scales,
//                K = 64) of each stage; a tcgen05.commit that arrives in both
//                CTAs releases ring stages and scale slots and signals the
//                accumulators;
//   warps 2..9   epilogue (both CTAs): tcgen05.ld of the CTA's 128 accumulator
//                rows (two warps per 32-lane quadrant), x alpha_a*alpha_b,
//                optional GELU(tanh), bf16 / fp32 stores;
//   warps 10..13 scale staging, one per 32-lane quadrant (both CTAs): each
//                stage's scale atoms from shared memory into registers, then
//                tcgen05.st into one of two 48-column scale slots, in the
//                layout the MMA reads (every quadrant holds all four 32-row
//                groups' scales; B scales for all 256 tile columns in each
//                CTA).  Keeping scale copies out of the MMA thread's in-order
//                tcgen05 queue lets the MMAs run back to back.
// Tensor memory (each CTA): the two scale slots at columns [0, 96),
// accumulator 0 at [96, 352) and accumulator 1 at [256, 512) -- the two share
// 96 columns, which the epilogue drains first and releases.
// Given workspace slabs, the tiles left for the schedule's last, partial
// round are cut along K into work units for the pairs that would idle; their
// fp32 partial tiles go to the slabs and split_reduce_kernel, launched next on
// the same stream, adds them in a fixed order and stores the output.
// Every wait is bounded (wall clock through %globaltimer); on a timeout the
// CTA records NVFP4_ERR_TIMEOUT in the device error word, drains what it
// issued and frees its tensor memory before returning.
#include <cuda.h>

#include "device_common.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

constexpr int BM = 128;           // rows per CTA (one TMEM lane per row); 256 per pair
constexpr int BN = 256;           // columns per tile; each CTA holds half of B
constexpr int BK = 256;           // K elements per stage = 128 bytes of codes per row
constexpr int BK_BYTES = BK / 2;  // one 128-byte swizzle row
constexpr int MMA_K = 64;         // K per tcgen05.mma (kind::mxf4nvf4)
constexpr int kStages = 5;
constexpr int kEpiWarps = 8;
constexpr int kSfWarps = 4;
constexpr int kSfWarp0 = 2 + kEpiWarps;  // first scale-staging warp
constexpr int kNumThreads = (2 + kEpiWarps + kSfWarps) * 32;
constexpr int kABytes = BM * BK_BYTES;          // 16 KB: this CTA's A rows
constexpr int kBBytes = (BN / 2) * BK_BYTES;    // 16 KB: this CTA's half of B
constexpr int kSfaBytes = 4 * 512;              // 4 atoms (128 rows x 16 blocks)
constexpr int kSfbBytes = (BN / 128) * 4 * 512; // both 128-row bands of the tile
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
// epilogue staging: per epilogue warp two buffers of a 32-row x 16-column
// output chunk (fp32 size), stored to global memory by TMA
constexpr int kEpiChunkBytes = 32 * 16 * 4;
constexpr int kEpiStageBytes = kEpiWarps * 2 * kEpiChunkBytes;
constexpr int kSmemBytes =
    kStages * kStageBytes + kEpiStageBytes + 1024 /*align*/ + 512 /*barriers*/;
// tensor memory columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfSlotCol = 0;   // two scale slots of 48 columns
constexpr uint32_t kAcc0Col = 96;    // accumulator 0 at column 96, 1 at 256
constexpr uint32_t kAcc1Col = 256;
constexpr uint32_t kOvlCols = 96;    // columns [256, 352) belong to both
constexpr uint32_t kSfSlotCols = 48; // A: 4 per MMA k-block (16), B: 8 per k-block (32)
constexpr int kSfSlots = 2;
constexpr int kGroupM = 8;           // tile raster: 8 M-tiles per group
// Pipeline waits give up after Params::wait_limit_ns (2 s unless the process
// set another bound with nvfp4_set_wait_limit); the waits of the exit path --
// copies in flight, the pair's last MMAs -- keep fixed bounds of their own, so
// even a very short pipeline bound leaves the CTA time to let everything it
// issued complete before it frees tensor memory and exits.
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s per copy in flight
constexpr uint64_t kMmaDoneLimitNs = 2000000000ull;  // 2 s for the last MMAs

// --------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// Arrive on a barrier of this CTA (release at CTA scope: prior shared-memory
// reads are complete before the stage can be refilled).
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Arrive on the leader CTA's copy of a barrier.  Only tensor-memory work is
// handed over this way (scale slots written, accumulator columns read), and
// that is ordered by tcgen05.fence::before_thread_sync on this side and
// tcgen05.fence::after_thread_sync on the waiting side, so the arrive itself
// is relaxed: a release at cluster scope would wait for this CTA's
// outstanding global stores and bulk copies, hundreds of nanoseconds.
__device__ __forceinline__ void mbar_arrive_leader(uint32_t local_bar, bool leader) {
  if (leader) {
    mbar_arrive(local_bar);
  } else {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(remote) : "r"(local_bar));
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote)
                 : "memory");
  }
}
// Reduces the byte count a barrier's current phase still waits for
// (accounts for copies that will never be issued).
__device__ __forceinline__ void mbar_complete_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Store into the leader CTA's copy of a shared-memory word, then arrive on
// the leader's copy of a barrier with release at cluster scope (the store is
// visible to a thread that then waits on the barrier with acquire).
__device__ __forceinline__ void store_and_arrive_leader(uint32_t local_word, uint32_t value,
                                                        uint32_t local_bar) {
  uint32_t rw, rb;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(rw) : "r"(local_word));
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(rb) : "r"(local_bar));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(rw), "r"(value) : "memory");
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(rb)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2; "
      "selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; returns false on timeout or when another role aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (abort_flag && *abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) return false;
    }
  }
}
// Bounded wait with acquire at cluster scope (no abort flag).
__device__ __forceinline__ bool mbar_wait_acq_cluster(uint32_t bar, uint32_t parity,
                                                      uint64_t limit_ns) {
  if (mbar_try_wait_acq_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    if ((i & 63) == 0 && globaltimer() - t0 > limit_ns) return false;
  }
}
// Tile load into this CTA's own shared memory, completion counted on a
// barrier of either CTA of the pair (2-SM form).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int32_t c0,
                                                 int32_t c1, uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(cluster_bar)
      : "memory");
}
// Tile store from this CTA's shared memory (dense box) to global memory;
// rows and columns outside the tensor are clipped.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t c0,
                                             int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          (uint64_t)map),
      "r"(src), "r"(c0), "r"(c1)
      : "memory");
}
// Untiled copy of `bytes` (a multiple of 16, both addresses 16-byte
// aligned) from this CTA's shared memory to global memory, in the bulk group.
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// at most one committed store group still reading its shared memory
__device__ __forceinline__ void bulk_wait_read_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrives on the barrier at this shared-memory offset in both CTAs of the pair
// once every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                            uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p; }" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// bf16 x bf16 -> fp32 MMA of a CTA pair (the LoRA branch), K = 16 per call.
__device__ __forceinline__ void tc_mma_pair_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t r[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// The load without its wait; the registers are valid only after tmem_wait16.
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t r[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// Waits for every tcgen05.ld of this thread (kWait) or only orders after an
// earlier wait; either way r passes through the statement, so no use of it is
// scheduled before the wait.
#define NVFP4_TIE16(r)                                                                        \
  "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),         \
      "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), \
      "+r"(r[14]), "+r"(r[15])
template <bool kWait>
__device__ __forceinline__ void tmem_wait16(uint32_t r[16]) {
  if constexpr (kWait)
    asm volatile("tcgen05.wait::ld.sync.aligned;" : NVFP4_TIE16(r) : : "memory");
  else
    asm volatile("" : NVFP4_TIE16(r) : : "memory");
}
#undef NVFP4_TIE16
// Tensor-memory stores of 16 consecutive 32-bit columns for the 32 lanes of
// this warp's quadrant (taddr carries the quadrant's first lane).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t r[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 format): start address >> 4 in
// bits 0-13, leading byte offset >> 4 in 16-29, stride byte offset >> 4 in
// 32-45, version 1 in 46-47, base offset 0, layout type in 61-63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
// K-major operand tile, 128-byte swizzle: rows of 128 bytes, 8-row groups
// 1024 bytes apart.
__device__ __forceinline__ uint64_t operand_desc(uint32_t addr) {
  return smem_desc(addr, 16, 1024, 2 /*SWIZZLE_128B*/);
}
// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (format 1), UE4M3
// scales (bit 23 = 0), K-major A and B, N >> 3 in bits 17-22, M >> 4 in
// bits 24-28, scale-factor ids 0.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Instruction descriptor, kind::f16 with bf16 A and B (format 1 in bits 7-9
// and 10-12), fp32 accumulation (bits 4-5 = 1), K-major A and B, N >> 3 in
// bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t instr_desc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// GELU(tanh form) in fp32: 0.5 y (1 + tanh(u)), u = sqrt(2/pi) (y + 0.044715
// y^3), evaluated as y * sigmoid(2u) = y / (1 + exp(-2u)) (the same function:
// 1 + tanh(u) = 2 / (1 + exp(-2u))), with exp(-2u) = 2^(y (c0 + c1 y^2)),
// c0 = -2 log2(e) sqrt(2/pi), c1 = 0.044715 c0, through the hardware ex2 and
// the __fdividef intrinsic.  For |2u| up to the point where the quotient
// saturates, the relative errors (the exponent's few ulp, scaled by its
// magnitude, a couple of ulp of ex2 and of the quotient) move the result by
// less than 2^-18 |y|; 2^(...) overflowing to +inf gives -0 (GELU of a large
// negative y is below any fp32 of its magnitude's scale), and __fdividef
// returning 0 for denominators above 2^126 does the same.  So
// |GELU_gpu(y) - GELU(y)| < 2^-17 |y| -- negligible against the GEMM's
// 1e-3 sum_k |a_k b_k|.
__device__ __forceinline__ float gelu_tanh(float y) {
  constexpr double kC0 = -2.0 * 1.4426950408889634 * 0.7978845608028654;
  const float c0 = (float)kC0, c1 = (float)(kC0 * 0.044715);
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(y * fmaf(c1, y * y, c0)));
  return __fdividef(y, 1.0f + e);
}

struct Params {
  const uint8_t* a_sf;
  const uint8_t* b_sf;
  const float* a_alpha;
  const float* b_alpha;
  void* out;
  int64_t ldo;
  int32_t M, N, K;
  int32_t out_bf16;
  int32_t epilogue;
  uint32_t* err;
  // non-null: each CTA writes the largest |stored value| of its tiles (after
  // the activation and the output rounding, rows past M excluded) to
  // amax_partials[blockIdx.x]; CTA 0 zeroes the slots of absent CTAs, so a
  // quantizer can reduce all kMaxAmaxCtas slots
  float* amax_partials;
  uint64_t wait_limit_ns;  // bound of each pipeline wait
  int32_t stall;           // test hook: the MMA issuer first waits on a barrier nothing completes
  // LoRA branch: lora_kt extra ring stages per tile after the FP4 stages,
  // each a 128-byte column chunk (64 bf16) of the scaled adapter input U'
  // [M, 2r] (hi and lo halves) and of B_lora [N, r] (chunk c mod lora_kt / 2)
  int32_t lora_kt;
  // Work units: [0, full_tiles) are whole tiles; each of the next tail_tiles
  // tiles is cut into split_s ranges of K stages, one unit per range, whose
  // fp32 partial sums go to slab (unit - full_tiles) of `slabs` for
  // split_reduce_kernel.  No split: full_tiles = all tiles, tail_tiles = 0,
  // split_s = 1.  A slab is 256 x 256 fp32 in 2 KB blocks of 32 rows x 16
  // columns (row-major inside), block (row / 32, column / 16) at
  // ((row / 32) * 16 + column / 16) * 2 KB: one epilogue staging chunk each.
  int32_t full_tiles, tail_tiles, split_s;
  float* slabs;
};

// Tile t of the grouped raster -> (tile row, tile column).
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int& mt, int& nt) {
  const int per_group = kGroupM * num_n;
  const int g = t / per_group;
  const int first_m = g * kGroupM;
  const int gm = min(kGroupM, num_m - first_m);
  const int r = t - g * per_group;
  mt = first_m + r % gm;
  nt = r / gm;
}

// Work unit u: its tile, its K stages [kt0, kt1) and its partial-sum slab
// (-1: a whole tile, stored to the output).
struct Unit {
  int tile, kt0, kt1, slab;
};
template <bool kSplit>
__device__ __forceinline__ Unit unit_of(const Params& p, int u, int num_kt, int total_kt) {
  Unit w;
  if (!kSplit || u < p.full_tiles) {
    w.tile = u;
    w.kt0 = 0;
    w.kt1 = total_kt;
    w.slab = -1;
  } else {
    const int v = u - p.full_tiles, i = v / p.split_s, j = v - i * p.split_s;
    w.tile = p.full_tiles + i;
    w.kt0 = j * num_kt / p.split_s;
    w.kt1 = (j + 1) * num_kt / p.split_s;
    w.slab = v;
  }
  return w;
}

// max(|a|, |b|) per bf16 half of two packed words (sign bits cleared).
__device__ __forceinline__ uint32_t absmax2_bf16(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a & 0x7FFF7FFFu), "r"(b & 0x7FFF7FFFu));
  return r;
}

// One lane's 16 accumulator columns -> x alpha_a*alpha_b, optional GELU ->
// its row of the warp's staging chunk (32 rows x 16 columns, dense).  With
// the output amax on (track) and the lane's row inside M, the largest
// |stored value| is folded into amax (bf16 outputs: as packed bf16 pairs).
__device__ __forceinline__ void stage16(const Params& p, uint8_t* chunk, int lane,
                                        const uint32_t r[16], float scale, bool track,
                                        uint32_t& amax) {
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v[i] = __fmul_rn(__uint_as_float(r[i]), scale);
    if ((p.epilogue & 0xF) == 1) v[i] = gelu_tanh(v[i]);
  }
  if (p.out_bf16) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    if (track) {
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = absmax2_bf16(amax, w[i]);
    }
    uint4* d4 = reinterpret_cast<uint4*>(chunk + lane * 32);
    d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else {
    if (track) {
      float m = __uint_as_float(amax);
#pragma unroll
      for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
      amax = __float_as_uint(m);
    }
    float4* d4 = reinterpret_cast<float4*>(chunk + lane * 64);
#pragma unroll
    for (int i = 0; i < 4; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

// A split unit's lane: its 16 unscaled fp32 sums as its row of the chunk.
__device__ __forceinline__ void stage16_raw(uint8_t* chunk, int lane, const uint32_t r[16]) {
  uint4* d4 = reinterpret_cast<uint4*>(chunk + lane * 64);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
}

// kSplit: the launch has split units (a separate instance, so that the
// common unsplit launch carries none of their code).
template <bool kSplit>
__global__ void __launch_bounds__(kNumThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmU,
                const __grid_constant__ CUtensorMap tmL, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = sA + kStages * kABytes;
  uint8_t* sSFA = sB + kStages * kBBytes;
  uint8_t* sSFB = sSFA + kStages * kSfaBytes;
  uint8_t* sEpi = sSFB + kStages * kSfbBytes;  // epilogue staging (1024-aligned)
  uint64_t* bars = (uint64_t*)(sEpi + kEpiStageBytes);
  uint64_t* full = bars;                      // [kStages] codes of both CTAs landed (leader)
  uint64_t* sf_in = full + kStages;           // [kStages] this CTA's scale atoms landed
  uint64_t* empty = sf_in + kStages;          // [kStages] stage free: MMAs done + scales read
  uint64_t* sf_full = empty + kStages;        // [2] scale slot written by both CTAs (leader)
  uint64_t* acc_full = sf_full + kSfSlots;    // [2] accumulator complete
  uint64_t* acc_empty = acc_full + 2;         // [2] accumulator drained by both CTAs (leader)
  uint64_t* ovl_free = acc_empty + 2;         // [1] shared columns drained by both (leader)
  uint64_t* mma_done = ovl_free + 1;          // [1] all MMAs of the pair done (leader)
  uint64_t* prod_end = mma_done + 1;          // [1] the peer's producer stopped (leader)
  uint64_t* never = prod_end + 1;             // [1] nothing arrives here (timeout test hook)
  uint32_t* tmem_slot = (uint32_t*)(never + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  uint32_t* cta_amax = (uint32_t*)(tmem_slot + 2);  // epilogue warps' output amax
  uint32_t* peer_it = tmem_slot + 3;  // stages the peer's producer issued (leader)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int num_m = (p.M + 2 * BM - 1) / (2 * BM), num_n = (p.N + BN - 1) / BN;
  const int num_kt = (p.K + BK - 1) / BK;
  const int total_kt = num_kt + p.lora_kt;  // FP4 stages, then the LoRA stages of a tile
  const int num_units = kSplit ? p.full_tiles + p.tail_tiles * p.split_s : num_m * num_n;
  const int kgroups = p.K / 64;  // 4-block scale groups per 128-row band
  const int mbands_total = (p.M + 127) / 128, nbands_total = (p.N + 127) / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&sf_in[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1 + kSfWarps);
    }
    for (int b = 0; b < kSfSlots; ++b) {
      mbar_init(smem_u32(&sf_full[b]), 2 * kSfWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 2 * kEpiWarps);
    }
    mbar_init(smem_u32(ovl_free), 2 * kEpiWarps);
    mbar_init(smem_u32(mma_done), 1);
    mbar_init(smem_u32(prod_end), 1);
    mbar_init(smem_u32(never), 1);
    *abort_flag = 0;
    *cta_amax = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  // both CTAs' barriers initialised and tensor memory allocated before any
  // cross-CTA arrival
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // operands may be written by the preceding kernel (programmatic launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = pair; u < num_units && ok; u += num_pairs) {
        const Unit w = unit_of<kSplit>(p, u, num_kt, total_kt);
        int mt, nt;
        tile_coords(w.tile, num_m, num_n, mt, nt);
        const int m0 = mt * 2 * BM + (int)rank * BM, nb0 = nt * BN + (int)rank * (BN / 2);
        const int mband = mt * 2 + (int)rank;
        for (int kt = w.kt0; kt < w.kt1; ++kt, ++it) {
          const int s = it % kStages;
          const uint32_t round = it / kStages;
          if (!mbar_wait(smem_u32(&empty[s]), (round & 1u) ^ 1u, abort_flag, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(smem_u32(&full[s]), 0);
          if (leader) mbar_expect_tx(smem_u32(&full[s]), 2 * (kABytes + kBBytes));
          if (kt >= num_kt) {
            // LoRA stage: 128-byte chunks of U' and B_lora, no scale atoms
            const int c = kt - num_kt;
            tma_load_2d_pair(smem_u32(sA + s * kABytes), &tmU, c * BK_BYTES, m0, fb);
            tma_load_2d_pair(smem_u32(sB + s * kBBytes), &tmL, (c % (p.lora_kt / 2)) * BK_BYTES,
                             nb0, fb);
            mbar_expect_tx(smem_u32(&sf_in[s]), 0u);
            continue;
          }
          tma_load_2d_pair(smem_u32(sA + s * kABytes), &tmA, kt * BK_BYTES, m0, fb);
          tma_load_2d_pair(smem_u32(sB + s * kBBytes), &tmB, kt * BK_BYTES, nb0, fb);
          const int atoms = min(4, kgroups - kt * 4);
          int nsf = mband < mbands_total ? 1 : 0;
          for (int h = 0; h < 2; ++h) nsf += (nt * 2 + h < nbands_total) ? 1 : 0;
          const uint32_t sb = smem_u32(&sf_in[s]);
          mbar_expect_tx(sb, (uint32_t)(atoms * 512 * nsf));
          if (mband < mbands_total)
            bulk_load(smem_u32(sSFA + s * kSfaBytes),
                      p.a_sf + ((int64_t)mband * kgroups + kt * 4) * 512, atoms * 512, sb);
          for (int h = 0; h < 2; ++h)
            if (nt * 2 + h < nbands_total)
              bulk_load(smem_u32(sSFB + s * kSfbBytes + h * 2048),
                        p.b_sf + ((int64_t)(nt * 2 + h) * kgroups + kt * 4) * 512, atoms * 512, sb);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.err, kDevErrTimeout);
      }
      // Every copy issued must have landed before the CTA retires (bounded
      // waits).  Stages before the last kStages issued were consumed by MMAs,
      // so they landed.  Scale atoms complete on this CTA's own barriers.
      for (uint32_t j = (it > (uint32_t)kStages ? it - kStages : 0u); j < it; ++j)
        mbar_wait(smem_u32(&sf_in[j % kStages]), (j / kStages) & 1u, nullptr, kDrainLimitNs);
      // Code tiles of both CTAs complete on the leader's barriers.  After an
      // abort the two producers may have stopped after different stage
      // counts (at most kStages apart: a stage is reissued only after the
      // MMAs consumed it from both CTAs), so the peer reports its count and
      // the leader re-balances each outstanding stage's expected bytes before
      // waiting: a stage only the peer loaded is armed for the peer's bytes, a
      // stage only the leader loaded is credited the peer's bytes that will
      // never come.
      if (!leader) {
        store_and_arrive_leader(smem_u32(peer_it), it, smem_u32(prod_end));
      } else {
        uint32_t it_peer = it;
        if (mbar_wait_acq_cluster(smem_u32(prod_end), 0, p.wait_limit_ns + 5 * kDrainLimitNs))
          it_peer = *reinterpret_cast<volatile uint32_t*>(peer_it);
        else
          atomicOr(p.err, kDevErrTimeout);
        const uint32_t half = kABytes + kBBytes;
        for (uint32_t j = it; j < it_peer; ++j) mbar_expect_tx(smem_u32(&full[j % kStages]), half);
        for (uint32_t j = it_peer; j < it; ++j) mbar_complete_tx(smem_u32(&full[j % kStages]), half);
        const uint32_t it_max = it > it_peer ? it : it_peer;
        for (uint32_t j = (it_max > (uint32_t)kStages ? it_max - kStages : 0u); j < it_max; ++j)
          mbar_wait(smem_u32(&full[j % kStages]), (j / kStages) & 1u, nullptr, kDrainLimitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (leader && lane == 0) {
      constexpr uint32_t idesc = instr_desc(2 * BM, BN);
      static_assert(kSfSlots == 2, "the issue loop alternates two scale slots");
      uint32_t it = 0, tile_i = 0;
      // ring position of stage `it` and the phase parities it waits for,
      // advanced incrementally (no division in the issue loop)
      uint32_t st = 0, st_ph = 0, slot = 0, slot_ph = 0;
      const uint64_t desc_a0 = operand_desc(smem_u32(sA)), desc_b0 = operand_desc(smem_u32(sB));
      const uint32_t t_sf0 = tmem + kSfSlotCol, t_sf1 = tmem + kSfSlotCol + kSfSlotCols;
      const int nmma_last = (p.K - (num_kt - 1) * BK) / MMA_K;
      bool ok = true;
      // test hook (nvfp4_set_test_stall): a wait that runs out after the
      // pipeline bound while the producers' first stages are in flight
      if (p.stall && !mbar_wait(smem_u32(never), 0, abort_flag, p.wait_limit_ns)) ok = false;
      for (int u = pair; u < num_units && ok; u += num_pairs, ++tile_i) {
        const Unit w = unit_of<kSplit>(p, u, num_kt, total_kt);
        const uint32_t b = tile_i & 1u, use = tile_i >> 1;
        // accumulator b drained by both CTAs' epilogues of tile_i - 2, and
        // the shared columns by those of tile_i - 1
        if (use > 0 && !mbar_wait(smem_u32(&acc_empty[b]), (use - 1) & 1u, abort_flag, p.wait_limit_ns)) {
          ok = false;
          break;
        }
        if (tile_i > 0 && !mbar_wait(smem_u32(ovl_free), (tile_i - 1) & 1u, abort_flag, p.wait_limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t_acc = tmem + (b ? kAcc1Col : kAcc0Col);
        for (int kt = w.kt0; kt < w.kt1; ++kt, ++it) {
          if (!mbar_wait(smem_u32(&full[st]), st_ph, abort_flag, p.wait_limit_ns) ||
              !mbar_wait(smem_u32(&sf_full[slot]), slot_ph, abort_flag, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors of this stage's tiles: the start-address field (bits
          // 0-13, address / 16) advances by the stage offset and by 32 bytes
          // (2 units) per MMA k-block; shared memory is below 256 KB, so the
          // field never carries into the next one
          const uint64_t da = desc_a0 + (uint64_t)(st * (kABytes >> 4));
          const uint64_t db = desc_b0 + (uint64_t)(st * (kBBytes >> 4));
          if (kt >= num_kt) {
            // LoRA stage: four bf16 MMAs (K = 16, 32 bytes of each row) into the
            // same accumulator, which the FP4 stages have initialised
            constexpr uint32_t idesc16 = instr_desc_bf16(2 * BM, BN);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc_mma_pair_bf16(t_acc, da + 2 * k, db + 2 * k, idesc16, 1u);
          } else {
            const int nmma = kt == num_kt - 1 ? nmma_last : 4;
            const uint32_t t_sf = slot ? t_sf1 : t_sf0;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              if (k < nmma)
                tc_mma_pair(t_acc, da + 2 * k, db + 2 * k, idesc, t_sf + 4 * k, t_sf + 16 + 8 * k,
                            (kt > w.kt0 || k > 0) ? 1u : 0u);
          }
          // one commit frees the ring stage and, for the scale warps, the
          // stage's scale slot (they wait on empty[] two stages back)
          tc_commit_pair(smem_u32(&empty[st]));
          if (++st == kStages) {
            st = 0;
            st_ph ^= 1u;
          }
          slot ^= 1u;
          slot_ph ^= slot == 0u ? 1u : 0u;
        }
        // signals both CTAs once this tile's MMAs (and everything before) completed
        tc_commit_pair(smem_u32(&acc_full[b]));
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.err, kDevErrTimeout);
      }
      // no MMA may still run when the pair frees its tensor memory (bounded)
      tc_commit_pair(smem_u32(mma_done));
      mbar_wait(smem_u32(mma_done), 0, nullptr, kMmaDoneLimitNs);
    }
  } else if (warp < kSfWarp0) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;        // 0..7
    const int quad = warp & 3;     // TMEM lanes 32*quad .. 32*quad+31
    const int half = e >> 2;       // 0 / 1: first / second half of each column range
    const float scale = __fmul_rn(*p.a_alpha, *p.b_alpha);
    uint8_t* my_stage = sEpi + e * 2 * kEpiChunkBytes;
    uint32_t tile_i = 0, chunk_i = 0;
    const bool want_amax = p.amax_partials != nullptr;
    uint32_t lane_amax = 0u;  // bf16x2 pair (bf16 out) or fp32 bits (fp32 out), both >= 0
    for (int u = pair; u < num_units; u += num_pairs, ++tile_i) {
      const Unit w = unit_of<kSplit>(p, u, num_kt, total_kt);
      const uint32_t b = tile_i & 1u, use = tile_i >> 1;
      int mt, nt;
      tile_coords(w.tile, num_m, num_n, mt, nt);
      const int m0 = mt * 2 * BM + (int)rank * BM, n0 = nt * BN;
      if (!mbar_wait(smem_u32(&acc_full[b]), use & 1u, abort_flag, p.wait_limit_ns)) {
        atomicOr(p.err, kDevErrTimeout);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t_acc = tmem + (b ? kAcc1Col : kAcc0Col) + ((uint32_t)(quad * 32) << 16);
      const bool quad_live = m0 + quad * 32 < p.M;  // warp-uniform
      // The columns shared with the other accumulator (tile columns 160..255
      // of accumulator 0, 0..95 of accumulator 1) go first, split between
      // the two warps of each quadrant: read into registers with one wait and
      // released at once, since the next tile's MMAs wait for them; then
      // staged and stored, then the rest.
      const int ovl_c0 = b ? 0 : 256 - (int)kOvlCols;
      const int rest_c0 = b ? (int)kOvlCols : 0;
      constexpr int kOvlPer = (int)kOvlCols / 2, kRestPer = (256 - (int)kOvlCols) / 2;
      static_assert(kOvlPer == 48, "three 16-column chunks of shared columns per warp");
      // each 16-column chunk goes through one of the warp's two staging
      // buffers and leaves as one TMA store (rows past M are clipped)
      auto store_chunk = [&](int c, const uint32_t r[16]) {
        uint8_t* chunk = my_stage + (chunk_i & 1u) * kEpiChunkBytes;
        if (lane == 0) bulk_wait_read_one();  // this buffer's previous store has read it
        __syncwarp();
        if (!kSplit || w.slab < 0)
          stage16(p, chunk, lane, r, scale, want_amax && m0 + quad * 32 + lane < p.M, lane_amax);
        else
          stage16_raw(chunk, lane, r);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (!kSplit || w.slab < 0)
            tma_store_2d(&tmOut, smem_u32(chunk), n0 + c, m0 + quad * 32);
          else  // the chunk is one 2 KB block of the unit's slab
            bulk_store(p.slabs + ((size_t)(w.slab * 8 + (int)rank * 4 + quad) * 16 + c / 16) * 512,
                       smem_u32(chunk), kEpiChunkBytes);
          bulk_commit();
        }
        ++chunk_i;
      };
      auto drain = [&](int c0, int ncols) {
#pragma unroll 1
        for (int c = c0; c < c0 + ncols; c += 16) {
          if (!quad_live || n0 + c >= p.N) continue;
          uint32_t r[16];
          tmem_ld16(t_acc + (uint32_t)c, r);
          store_chunk(c, r);
        }
      };
      const int oc = ovl_c0 + half * kOvlPer;
      uint32_t o0[16], o1[16], o2[16];
      if (quad_live) {
        tmem_ld16_async(t_acc + (uint32_t)oc, o0);
        tmem_ld16_async(t_acc + (uint32_t)(oc + 16), o1);
        tmem_ld16_async(t_acc + (uint32_t)(oc + 32), o2);
        tmem_wait16<true>(o0);
        tmem_wait16<false>(o1);
        tmem_wait16<false>(o2);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_leader(smem_u32(ovl_free), leader);
      if (quad_live) {
        if (n0 + oc < p.N) store_chunk(oc, o0);
        if (n0 + oc + 16 < p.N) store_chunk(oc + 16, o1);
        if (n0 + oc + 32 < p.N) store_chunk(oc + 32, o2);
      }
      drain(rest_c0 + half * kRestPer, kRestPer);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_leader(smem_u32(&acc_empty[b]), leader);
    }
    // every store has left shared memory and reached global memory
    if (lane == 0) bulk_wait_all();
    __syncwarp();
    if (want_amax) {
      // the CTA's output amax: lanes -> warp -> the eight epilogue warps
      const float m = p.out_bf16 ? fmaxf(__uint_as_float(lane_amax << 16),
                                         __uint_as_float(lane_amax & 0xFFFF0000u))
                                 : __uint_as_float(lane_amax);
      const uint32_t wm = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m));
      if (lane == 0) atomicMax(cta_amax, wm);
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
      if (e == 0 && lane == 0) {
        p.amax_partials[blockIdx.x] = __uint_as_float(*cta_amax);
        if (blockIdx.x == 0)
          for (int i = gridDim.x; i < kMaxAmaxCtas; ++i) p.amax_partials[i] = 0.0f;
      }
    }
  } else {
    // ------------------------------------------------------------ scale staging
    // Quadrant q's lanes get, per MMA k-block k of the stage: A columns
    // 4k + j = word j of row (lane) of the k-block's A atom (the four 32-row
    // groups' 4 scales each), B columns 16 + 8k + 4h + j = word j of row
    // (lane) of band h's atom.
    const int quad = warp & 3;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int u = pair; u < num_units && ok; u += num_pairs) {
      const Unit w = unit_of<kSplit>(p, u, num_kt, total_kt);
      for (int kt = w.kt0; kt < w.kt1; ++kt, ++it) {
        const int s = it % kStages;
        const uint32_t slot = it % kSfSlots;
        // The slot was last used by stage it - 2; its MMAs are done once that
        // stage's ring barrier completed its phase (the MMA commit and this
        // warp's own arrival).  That barrier cannot have moved on to its next
        // phase yet: that needs this warp's arrival for stage it + 3.
        const uint32_t prev = it - kSfSlots;
        if (!mbar_wait(smem_u32(&sf_in[s]), (it / kStages) & 1u, abort_flag, p.wait_limit_ns) ||
            (it >= (uint32_t)kSfSlots &&
             !mbar_wait(smem_u32(&empty[prev % kStages]), (prev / kStages) & 1u, abort_flag,
                        p.wait_limit_ns))) {
          ok = false;
          break;
        }
        if (kt >= num_kt) {
          // LoRA stage: no scales; hand the stage and the slot on unchanged
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(smem_u32(&empty[s]));
            mbar_arrive_leader(smem_u32(&sf_full[slot]), leader);
          }
          continue;
        }
        tc_fence_after();
        uint32_t ra[16], rb[32];
        const uint8_t* sfa = sSFA + s * kSfaBytes + 16 * lane;
        const uint8_t* sfb = sSFB + s * kSfbBytes + 16 * lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 a4 = *reinterpret_cast<const uint4*>(sfa + 512 * k);
          const uint4 b0 = *reinterpret_cast<const uint4*>(sfb + 512 * k);
          const uint4 b1 = *reinterpret_cast<const uint4*>(sfb + 2048 + 512 * k);
          ra[4 * k] = a4.x, ra[4 * k + 1] = a4.y, ra[4 * k + 2] = a4.z, ra[4 * k + 3] = a4.w;
          rb[8 * k] = b0.x, rb[8 * k + 1] = b0.y, rb[8 * k + 2] = b0.z, rb[8 * k + 3] = b0.w;
          rb[8 * k + 4] = b1.x, rb[8 * k + 5] = b1.y, rb[8 * k + 6] = b1.z, rb[8 * k + 7] = b1.w;
        }
        // the stage's scale bytes are in registers: the ring slot may refill
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
        const uint32_t t_sf = tmem + lane_addr + kSfSlotCol + slot * kSfSlotCols;
        tmem_st16(t_sf, ra);
        tmem_st16(t_sf + 16, rb);
        tmem_st16(t_sf + 32, rb + 16);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_leader(smem_u32(&sf_full[slot]), leader);
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(p.err, kDevErrTimeout);
    }
  }

  // ---------------------------------------------------------------- teardown
  // neither CTA frees its tensor memory or shared memory while the pair's
  // MMAs or the other CTA's arrivals may still touch them
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// The LoRA branch's adapter input, scaled into the accumulator's units: the
// epilogue multiplies the whole accumulator by a_alpha * b_alpha, so the
// bf16 MMAs must add u * c with c = scale / (a_alpha * b_alpha).  u * c (fp32)
// is split into hi = bf16(u c) and lo = bf16(u c - hi), written side by side
// as one [M, 2 rank] bf16 row each; hi + lo is within 2^-17 of u c, and the
// MMAs' products of bf16 values are exact in fp32.  One thread per 8
// consecutive elements of a row.
__global__ void __launch_bounds__(256)
    lora_prescale_kernel(const __nv_bfloat16* u, int64_t ldu, int64_t M, int64_t rank,
                         const float* a_alpha, const float* b_alpha, float scale,
                         __nv_bfloat16* out) {
  const float c = __fdiv_rn(scale, __fmul_rn(*a_alpha, *b_alpha));
  const int64_t groups = rank / 8, n = M * groups;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < n;
       g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = g / groups, j = (g - m * groups) * 8;
    const uint4 raw = *reinterpret_cast<const uint4*>(u + m * ldu + j);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = __fmul_rn(__uint_as_float(w[k] << 16), c);
      const float b = __fmul_rn(__uint_as_float(w[k] & 0xFFFF0000u), c);
      const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
      const float ha = __bfloat162float(h.x), hb = __bfloat162float(h.y);
      const __nv_bfloat162 l = __floats2bfloat162_rn(__fsub_rn(a, ha), __fsub_rn(b, hb));
      hi[k] = *reinterpret_cast<const uint32_t*>(&h);
      lo[k] = *reinterpret_cast<const uint32_t*>(&l);
    }
    __nv_bfloat16* row = out + m * 2 * rank;
    *reinterpret_cast<uint4*>(row + j) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(row + rank + j) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// --------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() { return (EncodeTiledFn)tensor_map_encoder(); }

// A matrix of `rows` rows of `row_bytes` bytes (row stride stride_bytes) as
// 128-byte x box_rows tiles, 128-byte swizzle, zero fill past the edges.
bool make_rows_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes,
                   int64_t stride_bytes, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)stride_bytes};
  cuuint32_t box[2] = {(cuuint32_t)BK_BYTES, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Codes [rows, K/2] bytes, box = 128 bytes x box_rows rows, 128-byte swizzle,
// out-of-bounds rows / columns read as zero.
bool make_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {(cuuint32_t)BK_BYTES, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void*)codes, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The split tiles: out = a_alpha b_alpha * (slab 0 + slab 1 + ... + slab S-1)
// of each, summed in slab order (fp32), then rounded to the output type as
// the GEMM's epilogue does; rows past M and columns past N are not stored.
// kReduceRows rows of a 256-column tile per block, four columns per thread.
constexpr int kReduceRows = 4;
__global__ void __launch_bounds__(kReduceRows * (BN / 4))
    split_reduce_kernel(const float* __restrict__ slabs, const Params p, int num_m, int num_n) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int kBlocksPerTile = 2 * BM / kReduceRows;
  const int i = blockIdx.x / kBlocksPerTile;
  const int r = (blockIdx.x % kBlocksPerTile) * kReduceRows + threadIdx.x / (BN / 4);
  const int c = (threadIdx.x % (BN / 4)) * 4;
  int mt, nt;
  tile_coords(p.full_tiles + i, num_m, num_n, mt, nt);
  const int m = mt * 2 * BM + r, n = nt * BN + c;
  if (m >= p.M || n >= p.N) return;  // N % 16 == 0: columns n .. n + 3 all inside
  // slab block (r / 32, c / 16), row r % 32, columns c % 16 .. + 3
  const float4* src = reinterpret_cast<const float4*>(
      slabs + (size_t)i * p.split_s * 2 * BM * BN + ((r / 32) * 16 + c / 16) * 512 + (r % 32) * 16 +
      c % 16);
  constexpr size_t kSlabF4 = (size_t)2 * BM * BN / 4;
  float4 acc = src[0];
  for (int j = 1; j < p.split_s; ++j) {
    const float4 v = src[j * kSlabF4];
    acc.x = __fadd_rn(acc.x, v.x);
    acc.y = __fadd_rn(acc.y, v.y);
    acc.z = __fadd_rn(acc.z, v.z);
    acc.w = __fadd_rn(acc.w, v.w);
  }
  const float scale = __fmul_rn(*p.a_alpha, *p.b_alpha);
  const float4 o = make_float4(__fmul_rn(acc.x, scale), __fmul_rn(acc.y, scale),
                               __fmul_rn(acc.z, scale), __fmul_rn(acc.w, scale));
  if (p.out_bf16) {
    __nv_bfloat162 h0 = __floats2bfloat162_rn(o.x, o.y), h1 = __floats2bfloat162_rn(o.z, o.w);
    uint2 w;
    w.x = *reinterpret_cast<uint32_t*>(&h0);
    w.y = *reinterpret_cast<uint32_t*>(&h1);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + (size_t)m * p.ldo + n) = w;
  } else {
    *reinterpret_cast<float4*>(static_cast<float*>(p.out) + (size_t)m * p.ldo + n) = o;
  }
}

cudaLaunchConfig_t pair_config(dim3 grid, cudaStream_t s, cudaLaunchAttribute attr[2]) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kNumThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cfg;
}

// Output [M, N] (bf16 or fp32, row stride ldo elements), box = 16 columns x
// 32 rows, dense in shared memory; stores clip at the tensor's edges.
bool make_out_map(CUtensorMap* map, void* out, int64_t M, int64_t N, int64_t ldo, bool bf16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t esz = bf16 ? 2 : 4;
  cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)ldo * esz};
  cuuint32_t box[2] = {16, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                  out, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Resident pairs: one pair per two SMs where the GPU's layout allows.
int max_resident_pairs() {
  static const int n_pairs = [] {
    if (cudaFuncSetAttribute(gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess)
      return 0;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = pair_config(dim3(2), nullptr, attr);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_kernel<false>, &cfg) != cudaSuccess || n < 1)
      n = num_sms() / 2;
    return n;
  }();
  return n_pairs;
}

// Split of the last, partial round of the persistent schedule: with `tiles`
// tiles on P resident pairs, the first tiles - tiles % P run whole; each of
// the rest is cut into S K ranges (S <= P / (tiles % P), at least
// kSplitMinStages stages each) run by otherwise idle pairs, so the launch
// ends after about tiles / P tile times instead of ceil(tiles / P).  Only
// for long K (a tile time worth more than the extra reduction launch), plain
// epilogues and no LoRA branch; at most slab_cap partial tiles.
constexpr int kSplitMinKt = 32;      // K >= 8192
constexpr int kSplitMinStages = 8;   // K stages per split unit
struct SplitPlan {
  int full_tiles, tail_tiles, split_s, pairs;
};
SplitPlan plan_split(int64_t M, int64_t N, int64_t K, bool eligible, int64_t slab_cap) {
  const int64_t tiles = ((M + 2 * BM - 1) / (2 * BM)) * ((N + BN - 1) / BN);
  const int64_t num_kt = (K + BK - 1) / BK;
  const int P = max_resident_pairs();
  SplitPlan sp{(int)tiles, 0, 1, (int)(tiles < P ? tiles : P)};
  if (!eligible || P < 2 || num_kt < kSplitMinKt) return sp;
  const int64_t rem = tiles % P;
  if (rem == 0) return sp;
  int64_t S = P / rem;
  if (S > num_kt / kSplitMinStages) S = num_kt / kSplitMinStages;
  if (S * rem > slab_cap) S = slab_cap / rem;
  if (S < 2) return sp;
  sp.full_tiles = (int)(tiles - rem);
  sp.tail_tiles = (int)rem;
  sp.split_s = (int)S;
  const int64_t units = sp.full_tiles + rem * S;
  sp.pairs = (int)(units < P ? units : P);
  return sp;
}

int launch_persistent(const GemmArgs& a, cudaStream_t s) {
  CUtensorMap tmA, tmB, tmOut, tmU, tmL;
  if (!make_out_map(&tmOut, a.out, a.M, a.N, a.ldo, a.out_bf16 != 0))
    return (int)cudaErrorInvalidValue;
  if (!make_codes_map(&tmA, a.a_codes, a.M, a.K, BM)) return (int)cudaErrorInvalidValue;
  if (!make_codes_map(&tmB, a.b_codes, a.N, a.K, BN / 2)) return (int)cudaErrorInvalidValue;
  int32_t lora_kt = 0;
  if (a.rank > 0) {
    // the scaled adapter input first (the GEMM waits for it: programmatic launch)
    const int64_t groups = a.M * (a.rank / 8);
    int64_t grid = (groups + 255) / 256;
    if (grid > (int64_t)num_sms() * 8) grid = (int64_t)num_sms() * 8;
    lora_prescale_kernel<<<(unsigned)(grid < 1 ? 1 : grid), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(a.lora_u), a.ldu, a.M, a.rank, a.a_alpha, a.b_alpha,
        a.lora_scale, static_cast<__nv_bfloat16*>(a.u_scaled));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
    if (!make_rows_map(&tmU, a.u_scaled, a.M, 4 * a.rank, 4 * a.rank, BM) ||
        !make_rows_map(&tmL, a.lora_b, a.N, 2 * a.rank, 2 * a.ldl, BN / 2))
      return (int)cudaErrorInvalidValue;
    lora_kt = (int32_t)(a.rank / 32);  // 2 rank bf16 of U' per row = rank / 32 chunks of 128 B
  } else {
    tmU = tmA;  // unused
    tmL = tmB;
  }
  Params p;
  p.a_sf = a.a_sf;
  p.b_sf = a.b_sf;
  p.a_alpha = a.a_alpha;
  p.b_alpha = a.b_alpha;
  p.out = a.out;
  p.ldo = a.ldo;
  p.M = (int32_t)a.M;
  p.N = (int32_t)a.N;
  p.K = (int32_t)a.K;
  p.out_bf16 = a.out_bf16;
  p.epilogue = a.epilogue;
  p.amax_partials = a.amax_partials;
  p.err = a.err;
  p.wait_limit_ns = a.wait_limit_ns;
  p.stall = a.stall;
  p.lora_kt = lora_kt;
  if (max_resident_pairs() < 1) return (int)cudaErrorInvalidConfiguration;
  const SplitPlan sp = plan_split(a.M, a.N, a.K, lora_kt == 0 && a.epilogue == 0 && a.slabs,
                                  a.slab_cap);
  p.full_tiles = sp.full_tiles;
  p.tail_tiles = sp.tail_tiles;
  p.split_s = sp.split_s;
  p.slabs = a.slabs;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_config(dim3(2 * sp.pairs), s, attr);
  cudaError_t e = sp.split_s > 1
                      ? cudaLaunchKernelEx(&cfg, gemm_kernel<true>, tmA, tmB, tmOut, tmU, tmL, p)
                      : cudaLaunchKernelEx(&cfg, gemm_kernel<false>, tmA, tmB, tmOut, tmU, tmL, p);
  if (e != cudaSuccess || sp.split_s == 1) return (int)e;
  // the split tiles' partial sums, added in slab order
  cudaLaunchConfig_t rc = {};
  rc.gridDim = dim3((unsigned)(sp.tail_tiles * (2 * BM / kReduceRows)));
  rc.blockDim = dim3(kReduceRows * (BN / 4));
  rc.stream = s;
  cudaLaunchAttribute rattr[1];
  rattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  rattr[0].val.programmaticStreamSerializationAllowed = 1;
  rc.attrs = rattr;
  rc.numAttrs = 1;
  const int num_m = (int)((a.M + 2 * BM - 1) / (2 * BM)), num_n = (int)((a.N + BN - 1) / BN);
  return (int)cudaLaunchKernelEx(&rc, split_reduce_kernel, (const float*)a.slabs, p, num_m, num_n);
}

}  // namespace

void* tensor_map_encoder() {
  static void* fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      ptr = nullptr;
    return ptr;
  }();
  return fn;
}

int launch_gemm(const GemmArgs& a, cudaStream_t s, bool* unsupported) {
  *unsupported = false;
  if (a.M > (int64_t)INT32_MAX / 2 || a.N > (int64_t)INT32_MAX / 2 || a.K > (int64_t)INT32_MAX / 2) {
    *unsupported = true;
    return 0;
  }
  return launch_persistent(a, s);
}

int64_t gemm_split_slabs(int64_t M, int64_t N, int64_t K, int32_t epilogue) {
  if (M < 1 || N < 1 || K < 64 || M > (int64_t)INT32_MAX / 2 || N > (int64_t)INT32_MAX / 2 ||
      K > (int64_t)INT32_MAX / 2)
    return 0;
  const SplitPlan sp = plan_split(M, N, K, epilogue == 0, INT64_MAX);
  return sp.split_s > 1 ? (int64_t)sp.tail_tiles * sp.split_s : 0;
}

}  // namespace nvfp4
