// SharQ linear layer GEMM (K3): structured-sparse + dense block-scaled FP4 MMAs into one
// tensor-memory accumulator, one epilogue.
//
// Per "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM Inference"
// (Abstract), the backbone goes through a sparse FP4 GEMM and the residual through a
// dense FP4 GEMM that makes up for what the mask dropped and for the backbone's
// quantization error; both read the same FP4 weight codes, each path with its own
// scale view. The README mirror ("Benchmarks") runs this path with the epilogue fused.
//
// sm_100a design. A cluster of two CTAs on the two SMs of a TPC works on one 256 x 256
// output tile with cta_group::2 MMAs (M = 256, N = 256): each CTA loads its own 128
// activation rows and half of the weight tile (128 rows), so every weight byte crosses
// into shared memory once per pair. Persistent over tiles, K steps of 256, four stages.
// Both operands are pre-tiled in global memory (chunks of 128 rows x 256 K that are the
// exact shared-memory image: swizzled codes, metadata, 128x4 scale atoms), so a stage is
// two bulk tensor copies per CTA -- the copy count per stage, not the bytes, is what
// bounds a TMA-fed pipeline at this tile size.
//   warp 0      TMA producer (both CTAs): the activation chunk and the weight chunk of the
//               K step; each CTA's loads complete on its own stage barrier.
//   warp 1      TMEM owner (both CTAs) and, in the leader, the single MMA-issuing thread:
//               two tcgen05.mma.sp (K=128 logical, pairwise 4:8) and four dense tcgen05.mma
//               (K=64) per K step accumulate into one fp32 accumulator of 128 x 256 per CTA.
//               Both paths carry the same per-row scale s_x, so one accumulator holds their
//               sum. Each weight chunk feeds both MMAs. Commits arrive on both CTAs'
//               barriers (multicast commit).
//   warps 2..9  epilogue (both CTAs): tcgen05.ld of the accumulator, y = acc * s_x[row] * s_w
//               rounded to bf16 in registers, the tensor memory handed back, then the block
//               staged in shared memory and written by bulk tensor stores (coalesced, clipped at
//               the tensor's edges) while the next tile's MMAs run. Row-wise 16-byte stores
//               from registers took a quarter of the kernel's time and delayed the next tile's
//               loads. (float32 output, a test format, is stored from registers.)
//   warps 10-13 scale writers (both CTAs, one tensor-memory lane quarter each): the K step's
//               scales and metadata from shared memory into registers and with tcgen05.st into
//               one of three tensor-memory buffers (every quarter holds each 32-row scale atom,
//               the layout the block-scaled MMA reads). tcgen05.cp copies issued by the leader
//               did the same but ran in order with the MMAs in the tensor pipe (~930 cycles
//               per K step against 768 of MMA work); the stores keep that pipe for the MMAs.
//               Each CTA's loads complete on its own stage barrier; the leader's MMA thread
//               waits for the writers of both CTAs.
// One launch may cover several problems of the same N and K (the experts of a mixture-of-
// experts layer): the persistent loop decodes each pair tile into (group, m-block, n-block)
// from a prefix table of tile counts. The kernel is launched as a programmatic dependent of
// the preparation and waits for it (griddepcontrol.wait) only after its prologue.
// Every mbarrier wait is bounded by a time limit; on expiry the CTA records a status word,
// stops issuing, drains (bounded) what it issued, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "sharq_common.cuh"
#include "sharq_internal.h"

namespace sharq {

__device__ uint32_t g_device_status = 0;  // bit 0: a bounded wait gave up

namespace {

constexpr int BM = 128;   // activation rows per CTA (256 per pair)
constexpr int BN = 256;   // output columns per pair tile
constexpr int BK = 256;   // logical K per stage
constexpr int kStagesPair = 4;  // pipeline stages of the pair form
constexpr int kStages1 = 3;     // of the single-CTA form (larger stages: both weight halves)
constexpr int kEpiWarps = 8;
constexpr int kSfWarps = 4;  // one per tensor-memory lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps + 32 * kSfWarps;  // producer, MMA, epilogue, scale writers
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 256;
constexpr uint32_t kScaleBufCols = 80;  // per buffer: meta 4, SFA_sp 8, SFA_res 16, SFB_sp 16, SFB_res 32
constexpr uint32_t kScaleBufs = 3;      // 256 + 3 * 80 = 496 of 512 columns
static_assert(kAccCols + kScaleBufs * kScaleBufCols <= kTmemCols, "tensor memory");
// Drains (own bulk copies and MMAs in flight before exit) always get the full bound, also when a
// test lowers the limit of the ordinary waits.
constexpr uint64_t kDrainLimitNs = 4000000000ull;

// shared-memory stage: the activation chunk, then the weight chunk (identical in both CTAs)
template <bool MX, bool SPARSE>
struct Stage {
  static constexpr ActTile A = act_tile(MX ? 1 : 0, 2, SPARSE);
  static constexpr WTile W = w_tile(MX ? 1 : 0);
  static constexpr int kW = A.bytes;  // 1024-aligned: the weight codes are 128-byte swizzled
  static constexpr int kBytes = A.bytes + W.bytes;
};
constexpr int kMaxStageBytes = 52224;  // NVFP4 SharQ: 29696 + 22528
// bf16 output staging for the epilogue's bulk tensor stores: per epilogue warp one box of 32
// rows x 32 columns (64-byte rows, 64-byte swizzle), reused four times per tile (on a pair's
// last tile the boxes go to the then idle pipeline stages instead, four per warp)
constexpr int kStageOutBytes = 2048;
constexpr int kOutOffsetPair = kStagesPair * kMaxStageBytes;  // 1024-aligned
constexpr int kSmemBytes = kOutOffsetPair + kEpiWarps * kStageOutBytes + 1024 /*align slack*/ + 256 /*barriers*/;
static_assert(Stage<false, true>::kBytes <= kMaxStageBytes && Stage<true, true>::kBytes <= kMaxStageBytes, "stage");
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kOutOffsetPair % 1024 == 0, "staging alignment");
static_assert(4 * kEpiWarps * kStageOutBytes <= kOutOffsetPair, "last-tile boxes fit in the pipeline stages");
// single-CTA form: a stage adds the other weight half's codes (128 rows x 128 bytes)
constexpr int kWCodeBytes = 16384;
constexpr int kMaxStage1Bytes = 52224 + kWCodeBytes;
constexpr int kOutOffset1 = kStages1 * kMaxStage1Bytes;
constexpr int kSmemBytes1 = kOutOffset1 + kEpiWarps * kStageOutBytes + 1024 + 256;
static_assert(Stage<false, true>::kBytes + kWCodeBytes <= kMaxStage1Bytes &&
                  Stage<true, true>::kBytes + kWCodeBytes <= kMaxStage1Bytes, "single-CTA stage");
static_assert(kSmemBytes1 <= 227 * 1024, "shared memory (single CTA)");
static_assert(kOutOffset1 % 1024 == 0 && 4 * kEpiWarps * kStageOutBytes <= kOutOffset1, "single-CTA staging");

struct __align__(64) TmaMaps {
  CUtensorMap act, w;  // both: rows of 1024 bytes (256 x u32), one box = one chunk
  CUtensorMap y;       // bf16 output [T][N], box 32 columns x 32 rows, 64-byte swizzle
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Arrive on a barrier given by its shared::cluster address (own or peer CTA), relaxed (no
// release ordering of this thread's memory operations): for handing back
// tensor memory whose loads have completed (tcgen05.wait::ld) -- nothing in memory is handed
// over, and a cluster-scope release was measured to stall the arriving thread ~1400 cycles.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// CLUSTER: acquire at cluster scope (the accumulator hand-back, arrived on from both CTAs);
// otherwise CTA scope (barriers completed by TMA transactions or tcgen05.commit).
template <bool CLUSTER>
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  if (CLUSTER)
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: gives up after `limit_ns` (or when another role of the CTA already
// gave up) and records the failure in the device status word.
template <bool CLUSTER = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          volatile uint32_t *abort_flag) {
  if (mbar_try<CLUSTER>(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try<CLUSTER>(bar, parity)) return true;
    if (i == 1 || (i & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) {
        *abort_flag = 1u;
        atomicOr(&g_device_status, 1u);
        return false;
      }
    }
  }
}

// The same wait in every lane of a warp, with a vote: the warp goes on only if every lane's
// wait succeeded, so it stays converged for the aligned tcgen05 instructions that follow even
// if lanes reached the time limit differently.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                               volatile uint32_t *abort_flag) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, limit_ns, abort_flag)) != 0;
}

// 2-D TMA load into this CTA's shared memory, completing on the barrier at `bar_cluster` (a
// shared::cluster address; the kernel passes this CTA's own stage barrier).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(bar_cluster)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// arrive once on the barrier at the same offset in both CTAs when this thread's MMAs finish
__device__ __forceinline__ void tc_commit_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

// commit to this CTA's barrier only (single-CTA form)
__device__ __forceinline__ void tc_commit_own(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
template <bool PAIR>
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  if (PAIR) tc_commit_both(bar);
  else tc_commit_own(bar);
}

template <bool PAIR>
__device__ __forceinline__ void tmem_alloc(uint32_t slot) {
  if (PAIR) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  } else {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
}
template <bool PAIR>
__device__ __forceinline__ void tmem_dealloc(uint32_t tmem) {
  if (PAIR) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  else asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}
// the pair's CTAs, or this CTA's threads
template <bool PAIR>
__device__ __forceinline__ void block_sync() {
  if (PAIR) cluster_sync();
  else __syncthreads();
}

// 2-D TMA load into this CTA's shared memory (single-CTA form: no cta_group qualifier)
__device__ __forceinline__ void tma_load_2d_1cta(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
// contiguous bytes from global into this CTA's shared memory (both 16-byte aligned, a multiple of
// 16 bytes), completing on `bar`
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// L2 prefetch of the 2-D box at (c0, c1) of a tensor map (no shared memory, no completion)
__device__ __forceinline__ void tma_prefetch_l2(const CUtensorMap *map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(c0), "r"(c1)
               : "memory");
}

// 2-D bulk tensor store from this CTA's shared memory (completion tracked by bulk groups)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(c0),
               "r"(c1), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until the committed stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// generic-proxy shared-memory writes become visible to the bulk-copy (async) proxy
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptors (K-major) as templates with the address field zero;
// layout 0 none, 2 SW128, 4 SW64; bit 46 is the sm_100 descriptor version. dsc() adds the
// 16-byte-unit address of one operand.
constexpr uint64_t desc_template(uint32_t sbo_bytes, uint32_t layout, uint32_t lbo_bytes) {
  return ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) | ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) |
         (1ull << 46) | ((uint64_t)layout << 61);
}
constexpr uint64_t kDescSw128 = desc_template(1024, 2, 16);  // 8-row groups of 128 B
constexpr uint64_t kDescSw64 = desc_template(512, 4, 16);    // 8-row groups of 64 B
__device__ __forceinline__ uint64_t dsc(uint64_t tmpl, uint32_t addr16) { return tmpl | (uint64_t)(addr16 & 0x3FFFu); }

// Instruction descriptor of the block-scaled MMA kinds (mxf4 / mxf4nvf4): E2M1 A and B,
// K-major, fp32 accumulate, M = 256 (two CTAs), N = 256.
__device__ __forceinline__ uint32_t idesc_bs(bool sparse, bool ue8m0, uint32_t sfa_id, uint32_t sfb_id,
                                             bool pair = true) {
  uint32_t d = 0;
  d |= (sparse ? 1u : 0u) << 2;
  d |= (sfb_id & 3u) << 4;
  d |= 1u << 7;                          // A format E2M1
  d |= 1u << 10;                         // B format E2M1
  d |= (uint32_t)(BN >> 3) << 17;        // N
  d |= (ue8m0 ? 1u : 0u) << 23;          // scale type: 0 UE4M3, 1 UE8M0
  d |= (uint32_t)((pair ? 2 * BM : BM) >> 4) << 24;  // M: 256 over the pair, or 128 on one CTA
  d |= (sfa_id & 3u) << 29;
  return d;
}

// Block-scaled FP4 MMAs, dense and structured-sparse, on the CTA pair (cta_group::2, M = 256)
// or on one CTA (cta_group::1, M = 128). The kind and block size follow the format.
#define SHARQ_MMA_DENSE(CG, KIND)                                                                              \
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"                                            \
               "tcgen05.mma.cta_group::" CG ".kind::" KIND " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem), \
               "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb))
#define SHARQ_MMA_SPARSE(CG, KIND)                                                                           \
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"                                          \
               "tcgen05.mma.sp.cta_group::" CG ".kind::" KIND " [%0], %1, %2, [%7], %3, [%5], [%6], p;\n\t}" ::"r"( \
                   d_tmem),                                                                                  \
               "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb), "r"(meta))

template <bool MX, bool PAIR = true>
__device__ __forceinline__ void mma_dense(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                          uint32_t sfb, uint32_t acc) {
  if (PAIR) {
    if (MX) SHARQ_MMA_DENSE("2", "mxf4.block_scale.block32");
    else SHARQ_MMA_DENSE("2", "mxf4nvf4.block_scale.block16");
  } else {
    if (MX) SHARQ_MMA_DENSE("1", "mxf4.block_scale.block32");
    else SHARQ_MMA_DENSE("1", "mxf4nvf4.block_scale.block16");
  }
}

template <bool MX, bool PAIR = true>
__device__ __forceinline__ void mma_sparse(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t meta, uint32_t idesc,
                                           uint32_t sfa, uint32_t sfb, uint32_t acc) {
  if (PAIR) {
    if (MX) SHARQ_MMA_SPARSE("2", "mxf4.block_scale.block32");
    else SHARQ_MMA_SPARSE("2", "mxf4nvf4.block_scale.block16");
  } else {
    if (MX) SHARQ_MMA_SPARSE("1", "mxf4.block_scale.block32");
    else SHARQ_MMA_SPARSE("1", "mxf4nvf4.block_scale.block16");
  }
}
#undef SHARQ_MMA_DENSE
#undef SHARQ_MMA_SPARSE

// 32 lanes x 32 columns of 32 bits; asynchronous until tmem_ld_wait()
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x N columns of 32 bits from registers (lane l writes r[0..N) to its lane)
__device__ __forceinline__ void tmem_st_x4(uint32_t taddr, const uint32_t *r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t *r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t *r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
               : "memory");
}
__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t *r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
               : "memory");
}
template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t *r) {
  if (N == 4) tmem_st_x4(taddr, r);
  if (N == 8) tmem_st_x8(taddr, r);
  if (N == 16) tmem_st_x16(taddr, r);
  if (N == 32) tmem_st_x32(taddr, r);
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// NA scale atoms (32 rows x 16 bytes each, at smem addresses base + atom_off(i)) into NA
// groups of 4 consecutive tensor-memory columns of this warp's lane quarter: lane l writes row
// l of every atom, so each quarter holds the whole atom (the replicated layout of the block-
// scaled MMA's scale factors).
template <int NA, typename F>
__device__ __forceinline__ void st_atoms(uint32_t taddr, uint32_t base, F atom_off, int lane) {
  uint32_t r[4 * NA];
#pragma unroll
  for (int i = 0; i < NA; ++i)
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[4 * i]), "=r"(r[4 * i + 1]), "=r"(r[4 * i + 2]), "=r"(r[4 * i + 3])
                 : "r"(base + atom_off(i) + lane * 16));
  tmem_st<4 * NA>(taddr, r);
}

// Orders every later use of r after the preceding tmem_ld_wait(): the registers written by
// an asynchronous tensor-memory load are only valid once the wait has returned.
__device__ __forceinline__ void reg_fence32(uint32_t *r) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// Group of a pair tile (groups hold consecutive tile ranges; empty groups are skipped).
template <int MAXG>
__device__ __forceinline__ int group_of(const GemmParams &p, int tile) {
  int g = 0;
  if (MAXG > 1)
    while (g + 1 < p.n_groups && tile >= p.grp[g + 1].tile_begin) ++g;
  return g;
}

template <int MAXG>
struct __align__(64) TmaMapSet {
  TmaMaps m[MAXG];
};
static_assert(sizeof(TmaMapSet<kMaxGroups>) + sizeof(GemmParams) <= 32764, "kernel parameter space");

// MAXG: 1 for one problem per launch, kMaxGroups for the grouped (mixture-of-experts) form.
// PAIR: the CTA-pair form (cta_group::2, 256 x 256 tiles); otherwise one CTA per 128 x 256
// tile (cta_group::1), for launches whose row groups are mostly at most 128 rows.
template <bool MX, bool SPARSE, int MAXG, bool PAIR>
__device__ __forceinline__ void gemm_body(const TmaMapSet<MAXG> &ms, const GemmParams &p) {
  constexpr int kStages = PAIR ? kStagesPair : kStages1;
  constexpr int kOutOffset = PAIR ? kOutOffsetPair : kOutOffset1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOutOffset + kEpiWarps * kStageOutBytes);
  // bars: full[kStages], empty[kStages], acc_full, acc_empty, drain, sf_full[kStages], sf_free[kScaleBufs]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * kStages + 3 + kScaleBufs);
  volatile uint32_t *abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const uint32_t smem0 = smem_u32(smem);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * kStages), acc_empty = acc_full + 8, drain_bar = acc_full + 16;
  auto sf_full_bar = [&](int s) { return bar0 + 8u * (2 * kStages + 3 + s); };
  auto sf_free_bar = [&](uint32_t b) { return bar0 + 8u * (3 * kStages + 3 + b); };

  using L = Stage<MX, SPARSE>;
  constexpr int apt_res = atoms_res(MX ? 1 : 0), apt_sp = atoms_sp(MX ? 1 : 0);
  // single-CTA stage: activation chunk, the two weight halves' codes back to back (one 256-row
  // B operand), then the weight scales (both halves' atoms, as the pair form's chunk has them)
  constexpr int kStageBytes = PAIR ? L::kBytes : L::kBytes + kWCodeBytes;
  constexpr int kWScales = PAIR ? L::kW : L::kW + kWCodeBytes;  // the weight scale region's base
  const int ks_total = p.K / BK;  // K steps per operand row block: the chunk stride
  const int num_tiles = p.num_tiles;
  // work units: CTA pairs, or single CTAs
  const int pair = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int num_pairs = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const uint64_t limit = p.wait_limit > 0 ? (uint64_t)p.wait_limit : 4000000000ull;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, (PAIR ? 2 : 1) * kEpiWarps);
    mbar_init(drain_bar, 1);
    for (int s = 0; s < kStages; ++s) mbar_init(sf_full_bar(s), (PAIR ? 2 : 1) * kSfWarps);  // writers of both CTAs
    for (uint32_t b = 0; b < kScaleBufs; ++b) mbar_init(sf_free_bar(b), 1);
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&ms.m[0].act) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&ms.m[0].w) : "memory");
  }
  if (warp == 1) tmem_alloc<PAIR>(smem_u32(tmem_slot));
  tc_fence_before();
  block_sync<PAIR>();  // barriers initialized and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0 && lane == 0 && pair < num_tiles) {
    // The packed weight is not an output of the preparation: its first K steps for this CTA's
    // first tile are fetched into L2 while the preparation may still be running.
    const int g = group_of<MAXG>(p, pair), lt = pair - p.grp[g].tile_begin;
    for (int h = 0; h < (PAIR ? 1 : 2); ++h) {
      const int w_row0 =
          (((lt / p.grp[g].num_m) * BN / 128 + (PAIR ? (int)rank : h)) * ks_total + p.grp[g].k0) * (L::W.bytes / 1024);
      for (int kt = 0; kt < kStages && kt < p.grp[g].num_k; ++kt)
        tma_prefetch_l2(&ms.m[g].w, 0, w_row0 + kt * (L::W.bytes / 1024));
    }
  }
  // Launched as a programmatic dependent of the preparation: the prologue above overlaps its
  // tail; its outputs are read only after it has completed and flushed.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, last_parity = 0;  // bit s: stage s armed / its last phase parity
      bool ok = true;
      const uint32_t full_own0 = PAIR ? map_to_rank(full_bar(0), rank) : full_bar(0);
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        const int g = group_of<MAXG>(p, tile), lt = tile - p.grp[g].tile_begin, num_m = p.grp[g].num_m;
        const TmaMaps &maps = ms.m[g];
        const int m0 = PAIR ? (lt % num_m) * (2 * BM) + (int)rank * BM : (lt % num_m) * BM;  // this CTA's rows
        const int n0 = (lt / num_m) * BN;  // the tile's output columns
        // chunk rows of 1024 bytes; the group's K steps start at k0
        const int a_row0 = ((m0 / 128) * ks_total + p.grp[g].k0) * (L::A.bytes / 1024);
        const int w_row0 = ((n0 / 128 + (int)rank) * ks_total + p.grp[g].k0) * (L::W.bytes / 1024);
        const int num_k = p.grp[g].num_k;
        // single CTA: the weight chunks of both 128-row halves, by plain bulk copies
        const uint8_t *w_half0 = p.grp[g].w_tiles + ((size_t)(n0 / 128) * ks_total + p.grp[g].k0) * L::W.bytes;
        const uint8_t *w_half1 = w_half0 + (size_t)ks_total * L::W.bytes;
        for (int kt = 0; kt < num_k; ++kt) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, limit, abort_flag)) { ok = false; break; }
          const uint32_t st = smem0 + stage * kStageBytes;
          // each CTA's loads complete on its own barrier: its scale writers wait for it, and
          // the leader's MMA learns of the peer's bytes through the peer's writers
          mbar_expect_tx(full_bar(stage), kStageBytes);
          armed |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          const uint32_t fb = full_own0 + 8u * stage;
          if (PAIR) {
            tma_load_2d(st, &maps.act, 0, a_row0 + kt * (L::A.bytes / 1024), fb);
            tma_load_2d(st + L::kW, &maps.w, 0, w_row0 + kt * (L::W.bytes / 1024), fb);
          } else {
            tma_load_2d_1cta(st, &maps.act, 0, a_row0 + kt * (L::A.bytes / 1024), fb);
            const size_t wk = (size_t)kt * L::W.bytes;
            bulk_load(st + L::kW, w_half0 + wk, kWCodeBytes, fb);
            bulk_load(st + L::kW + kWCodeBytes, w_half1 + wk, kWCodeBytes, fb);
            bulk_load(st + kWScales + kWCodeBytes, w_half0 + wk + kWCodeBytes, L::W.bytes - kWCodeBytes, fb);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // Drain before exit: every phase this CTA armed completes (its loads have landed).
        for (int s = 0; s < kStages; ++s)
          if (armed & (1u << s)) {
            volatile uint32_t no_abort = 0;
            mbar_wait(full_bar(s), (last_parity >> s) & 1u, kDrainLimitNs, &no_abort);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader CTA)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0, buf = 0;
      bool ok = true;
      const uint32_t acc = tmem;  // lanes 0..127 of each CTA, columns 0..255
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        // released by both CTAs' epilogue warps (remote arrives): cluster-scope acquire
        if (!mbar_wait<true>(acc_empty, acc_phase ^ 1u, limit, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const int num_k = p.grp[group_of<MAXG>(p, tile)].num_k;
        for (int kt = 0; kt < num_k; ++kt) {
          // the scale writers of both CTAs waited for their stage's bytes, then wrote its scales
          // (remote arrives: cluster-scope acquire)
          if (!mbar_wait<true>(sf_full_bar(stage), phase, limit, abort_flag)) { ok = false; break; }
          if (!mbar_wait(full_bar(stage), phase, limit, abort_flag)) { ok = false; break; }
          tc_fence_after();
          // descriptors: constant templates plus the operand's shared-memory address >> 4
          const uint32_t st4 = (smem0 + stage * kStageBytes) >> 4;
          const uint32_t sbuf = tmem + kAccCols + buf * kScaleBufCols;
          const uint32_t t_meta = sbuf, t_sfa_sp = sbuf + 4, t_sfa_res = sbuf + 12, t_sfb_sp = sbuf + 28,
                         t_sfb_res = sbuf + 44;
          constexpr int kA = 0, kW = L::kW;
          uint32_t accumulate = kt > 0 ? 1u : 0u;
          if (SPARSE) {
            // two sparse MMAs: 128 logical K each = 32 bytes of compressed A, 64 bytes of B
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              // NVFP4: 4 scales per row per MMA (one atom, id 0); MXFP4: 2 (half an atom)
              const uint32_t atom = MX ? (uint32_t)(j >> 1) : (uint32_t)j;
              const uint32_t id = MX ? (uint32_t)(2 * (j & 1)) : 0u;
              mma_sparse<MX, PAIR>(acc, dsc(kDescSw64, st4 + (kA + L::A.sp + 32 * j) / 16),
                                   dsc(kDescSw128, st4 + (kW + L::W.b + 64 * j) / 16), t_meta + 2 * j,
                                   idesc_bs(true, MX, id, id, PAIR), (t_sfa_sp + 4 * atom) | (id << 30),
                                   (t_sfb_sp + 8 * atom) | (id << 30), accumulate);
              accumulate = 1u;
            }
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // four dense MMAs of K = 64 (32 bytes of A and B)
            const uint32_t atom = MX ? (uint32_t)(j >> 1) : (uint32_t)j;
            const uint32_t id = MX ? (uint32_t)(2 * (j & 1)) : 0u;
            mma_dense<MX, PAIR>(acc, dsc(kDescSw128, st4 + (kA + L::A.res + 32 * j) / 16),
                                dsc(kDescSw128, st4 + (kW + L::W.b + 32 * j) / 16), idesc_bs(false, MX, id, id, PAIR),
                                (t_sfa_res + 4 * atom) | (id << 30), (t_sfb_res + 8 * atom) | (id << 30), accumulate);
            accumulate = 1u;
          }
          tc_commit<PAIR>(empty_bar(stage));  // frees the stage in both CTAs once these MMAs have read it
          tc_commit<PAIR>(sf_free_bar(buf));  // and the scale buffer in both CTAs
          if (++buf == kScaleBufs) buf = 0;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit<PAIR>(acc_full);
        acc_phase ^= 1u;
      }
      // Drain: all MMAs issued above complete before TMEM is released.
      tc_commit<PAIR>(drain_bar);
      volatile uint32_t no_abort = 0;
      mbar_wait(drain_bar, 0, kDrainLimitNs, &no_abort);
    }
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------------------------------------ epilogue (warps 2..9, both CTAs)
    const int quarter = warp & 3;          // TMEM lane quarter this warp may access
    const int col_half = (warp - 2) >> 2;  // columns [128*col_half, 128*col_half + 128)
    const int r_local = quarter * 32 + lane;
    const uint32_t acc_empty_leader = PAIR ? map_to_rank(acc_empty, 0) : acc_empty;
    const uint32_t out_smem = smem0 + kOutOffset + (warp - 2) * kStageOutBytes;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs) {
      const int g = group_of<MAXG>(p, tile), lt = tile - p.grp[g].tile_begin, num_m = p.grp[g].num_m;
      const GemmGroup &G = p.grp[g];
      const float s_w = G.tensor_scale[0];
      const int m0 = PAIR ? (lt % num_m) * (2 * BM) + (int)rank * BM : (lt % num_m) * BM, n0 = (lt / num_m) * BN;
      const int row = m0 + r_local;
      const float scale = row < G.T ? __fmul_rn(G.row_scale[row], s_w) : 0.f;
      if (!mbar_wait_warp(acc_full, acc_phase, limit, abort_flag)) break;
      tc_fence_after();
      const uint32_t tacc = tmem + ((uint32_t)(quarter * 32) << 16) + col_half * 128;
      const int col0 = n0 + col_half * 128;
      const bool row_ok = row < G.T;
      if (p.out_f32) {
        // float32 output: 32 columns at a time, the tensor memory held until the last load
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32_async(tacc + 32 * c, r);
          tmem_ld_wait();
          reg_fence32(r);
          const int col = col0 + 32 * c;
          if (!row_ok || col >= p.N) continue;
          float *dst = reinterpret_cast<float *>(G.y) + (size_t)row * p.N + col;
          if (col + 32 <= p.N) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4 *>(dst + i) =
                  make_float4(__fmul_rn(__uint_as_float(r[i]), scale), __fmul_rn(__uint_as_float(r[i + 1]), scale),
                              __fmul_rn(__uint_as_float(r[i + 2]), scale), __fmul_rn(__uint_as_float(r[i + 3]), scale));
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col + i < p.N) dst[i] = __fmul_rn(__uint_as_float(r[i]), scale);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty_leader);
      } else {
        // bf16 output: this warp's 32 rows x 128 columns are read and rounded (64 registers
        // of packed pairs), the tensor memory is handed back as soon as the last load has
        // landed, and the stores overlap the next tile's MMAs
        uint32_t packed[4][16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // two loads in flight per wait
          uint32_t r[2][32];
          tmem_ld32_async(tacc + 64 * h, r[0]);
          tmem_ld32_async(tacc + 64 * h + 32, r[1]);
          tmem_ld_wait();
          reg_fence32(r[0]);
          reg_fence32(r[1]);
          if (h == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty_leader);
          }
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              // packed product (round to nearest per lane; it feeds only the bf16 conversion)
              float y0 = __uint_as_float(r[c][2 * i]), y1 = __uint_as_float(r[c][2 * i + 1]);
              asm("{\n\t.reg .b64 x, s, z;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 s, {%2, %2};\n\t"
                  "mul.rn.f32x2 z, x, s;\n\tmov.b64 {%0, %1}, z;\n\t}"
                  : "+f"(y0), "+f"(y1)
                  : "f"(scale));
              const __nv_bfloat162 v = __floats2bfloat162_rn(y0, y1);
              packed[2 * h + c][i] = *reinterpret_cast<const uint32_t *>(&v);
            }
        }
        // Write this warp's 32 x 128 block with bulk tensor stores (coalesced; rows >= T and
        // columns >= N clipped by the tensor map) through 2 KB staging boxes of 32 x 32, in
        // 64-byte-swizzled rows: 16-byte unit u of row r at u ^ ((r / 2) % 4), conflict-free.
        // One box buffer per warp while MMAs may still read the pipeline stages; on the pair's
        // last tile every MMA has completed, so the stages' shared memory holds four boxes per
        // warp and the stores go out back to back.
        const int row0 = m0 + quarter * 32;
        const bool last = tile + num_pairs >= num_tiles;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t box = last ? smem0 + (uint32_t)(((warp - 2) * 4 + c) * kStageOutBytes) : out_smem;
          if (!last) {
            if (lane == 0) bulk_wait_read();  // the previous box has been read out of the buffer
            __syncwarp();
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t dst = box + lane * 64 + ((u ^ ((lane >> 1) & 3)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(packed[c][4 * u]),
                         "r"(packed[c][4 * u + 1]), "r"(packed[c][4 * u + 2]), "r"(packed[c][4 * u + 3])
                         : "memory");
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            if (row0 < G.T && col0 + 32 * c < p.N) tma_store_2d(&ms.m[g].y, box, col0 + 32 * c, row0);
            bulk_commit();
          }
        }
      }
      acc_phase ^= 1u;
    }
    // the stores have read their boxes before the CTA's shared memory goes away (they complete
    // in global memory before the grid does)
    if (lane == 0) bulk_wait_read();
  }

  else {
    // ------------------------------------------------------------ scale writers (warps 10..13, both CTAs)
    // Each warp writes the K step's scale factors and metadata into its lane quarter of one of
    // three tensor-memory buffers with tcgen05.st (registers -> tensor memory), so these writes
    // stay out of the tensor pipe that runs the MMAs in order.
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t sf_full_leader0 = PAIR ? map_to_rank(sf_full_bar(0), 0) : sf_full_bar(0);
    int stage = 0;
    uint32_t phase = 0, buf = 0, buf_phase = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
      const int num_k = p.grp[group_of<MAXG>(p, tile)].num_k;
      for (int kt = 0; kt < num_k; ++kt) {
        if (!mbar_wait_warp(full_bar(stage), phase, limit, abort_flag)) { ok = false; break; }
        // the buffer is free once the MMAs that last read it (kScaleBufs steps ago) completed
        if (!mbar_wait_warp(sf_free_bar(buf), buf_phase ^ 1u, limit, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = smem0 + stage * kStageBytes;
        const uint32_t sbuf = tmem + ((uint32_t)(quarter * 32) << 16) + kAccCols + buf * kScaleBufCols;
        const uint32_t t_meta = sbuf, t_sfa_sp = sbuf + 4, t_sfa_res = sbuf + 12, t_sfb_sp = sbuf + 28,
                       t_sfb_res = sbuf + 44;
        constexpr int kA = 0;
        // weight scales: the chunk holds the atoms of both 128-row halves of the pair's 256
        // columns (half 0, then half 1); in tensor memory they alternate per atom
        st_atoms<2 * apt_res>(t_sfb_res, st + kWScales + L::W.sf_res,
                              [&](int i) { return ((i & 1) * apt_res + (i >> 1)) * 512; }, lane);
        if (SPARSE)
          st_atoms<2 * apt_sp>(t_sfb_sp, st + kWScales + L::W.sf_sp,
                               [&](int i) { return ((i & 1) * apt_sp + (i >> 1)) * 512; }, lane);
        st_atoms<apt_res>(t_sfa_res, st + kA + L::A.sf_res, [&](int i) { return i * 512; }, lane);
        if (SPARSE) {
          st_atoms<apt_sp>(t_sfa_sp, st + kA + L::A.sf_sp, [&](int i) { return i * 512; }, lane);
          // metadata: 128 rows x 16 bytes, row r in lane r (not replicated)
          st_atoms<1>(t_meta, st + kA + L::A.meta + quarter * 32 * 16, [&](int) { return 0; }, lane);
        }
        // The stores have completed in this SM's tensor memory (wait::st) before the arrive
        // leaves; the MMA that reads them is issued only after the leader has seen all eight
        // arrives. Nothing in the memory hierarchy sits between the two, so the arrive is
        // relaxed: a cluster-scope release arrive stalled each writer ~1400 cycles per K step,
        // which made the writers, not the MMAs, set the pace (54 us against 35 us per launch).
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(sf_full_leader0 + 8u * stage);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
        if (++buf == kScaleBufs) { buf = 0; buf_phase ^= 1u; }
      }
    }
  }

  // Both CTAs: the leader arrives here only after its MMAs drained, so neither CTA frees
  // tensor memory the pair's MMAs still write, and no remote arrive targets an exited CTA.
  // The roles above run on lane 0 of their warps: each warp converges before the aligned
  // cluster barrier.
  __syncwarp();
  tc_fence_before();
  block_sync<PAIR>();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<PAIR>(tmem);
}

template <bool MX, bool SPARSE, int MAXG>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    sharq_gemm_kernel(const __grid_constant__ TmaMapSet<MAXG> ms, const __grid_constant__ GemmParams p) {
  gemm_body<MX, SPARSE, MAXG, true>(ms, p);
}

// One CTA per 128 x 256 tile (no cluster).
template <bool MX, bool SPARSE, int MAXG>
__global__ void __launch_bounds__(kThreads, 1)
    sharq_gemm1_kernel(const __grid_constant__ TmaMapSet<MAXG> ms, const __grid_constant__ GemmParams p) {
  gemm_body<MX, SPARSE, MAXG, false>(ms, p);
}

// ---------------------------------------------------------------- tensor-core peak loop
// The MMAs of one K step of the kernel above, issued back to back against one shared-memory
// stage and one tensor-memory scale buffer that stay resident: no loads, no scale writes, no
// epilogue. A launch on every SM pair measures the rate of the tensor pipe for this exact
// instruction mix, the ceiling the GEMM is compared with. MODE 0: the four dense MMAs of a K
// step; 1: the two sparse MMAs; 2: both (the SharQ K step). Operands are pseudo-random E2M1
// codes (every nibble is a value), block scales in [1/4, 4] and metadata of valid ascending
// pair indices; the accumulator restarts every 16 K steps, as the GEMM's does at K = 4096.
constexpr int kPeakThreads = 128;
constexpr int kPeakSmemBytes = kMaxStageBytes + 64 + 1024;

__device__ __forceinline__ uint32_t hash32(uint32_t x) {  // integer finalizer (xorshift-multiply)
  x ^= x >> 16;
  x *= 0x7feb352du;
  x ^= x >> 15;
  x *= 0x846ca68bu;
  x ^= x >> 16;
  return x;
}

template <bool MX, int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPeakThreads, 1)
    mma_peak_kernel(int iters, unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kMaxStageBytes);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 1);
  using L = Stage<MX, true>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t smem0 = smem_u32(smem), done = smem_u32(bars);

  for (int i = threadIdx.x; i < L::kBytes / 4; i += blockDim.x)
    reinterpret_cast<uint32_t *>(smem)[i] = hash32((uint32_t)i * 2654435761u + rank);
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  fence_proxy_async();  // the MMAs read the operands through the async proxy
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  {
    // scale buffer 0 (columns 256..335) of this warp's lane quarter: metadata in the first 4
    // columns, scale bytes in the rest
    const uint32_t base = tmem + ((uint32_t)(warp * 32) << 16) + kAccCols;
    // valid (i0 < i1) nibbles i0 | i1 << 2: 4 8 C 9 D E, two of them twice, packed 4 bits each
    constexpr uint32_t kMetaNibbles = 0xE4ED9C84u;
#pragma unroll 1
    for (int c = 0; c < (int)kScaleBufCols; c += 16) {
      uint32_t r[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t h = hash32((uint32_t)((warp * 32 + lane) * kScaleBufCols + c + j) ^ (rank << 20));
        uint32_t w = 0u;
        if (c + j < 4) {
#pragma unroll
          for (int n = 0; n < 8; ++n) w |= ((kMetaNibbles >> (4 * ((h >> (3 * n)) & 7u))) & 0xFu) << (4 * n);
        } else {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t hb = h >> (8 * b);
            const uint32_t code = MX ? 125u + (hb & 3u) + ((hb >> 2) & 1u) : ((5u + (hb & 3u)) << 3) | ((hb >> 2) & 7u);
            w |= code << (8 * b);
          }
        }
        r[j] = w;
      }
      tmem_st<16>(base + c, r);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (rank == 0 && warp == 1 && lane == 0) {
    const uint32_t st4 = smem0 >> 4;
    const uint32_t sbuf = tmem + kAccCols;
    const uint32_t t_meta = sbuf, t_sfa_sp = sbuf + 4, t_sfa_res = sbuf + 12, t_sfb_sp = sbuf + 28,
                   t_sfb_res = sbuf + 44;
    constexpr int kA = 0, kW = L::kW;
    for (int it = 0; it < iters; ++it) {
      uint32_t accumulate = (it & 15) ? 1u : 0u;
      if (MODE != 0) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t atom = MX ? (uint32_t)(j >> 1) : (uint32_t)j;
          const uint32_t id = MX ? (uint32_t)(2 * (j & 1)) : 0u;
          mma_sparse<MX>(tmem, dsc(kDescSw64, st4 + (kA + L::A.sp + 32 * j) / 16),
                         dsc(kDescSw128, st4 + (kW + L::W.b + 64 * j) / 16), t_meta + 2 * j,
                         idesc_bs(true, MX, id, id), (t_sfa_sp + 4 * atom) | (id << 30),
                         (t_sfb_sp + 8 * atom) | (id << 30), accumulate);
          accumulate = 1u;
        }
      }
      if (MODE != 1) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t atom = MX ? (uint32_t)(j >> 1) : (uint32_t)j;
          const uint32_t id = MX ? (uint32_t)(2 * (j & 1)) : 0u;
          mma_dense<MX>(tmem, dsc(kDescSw128, st4 + (kA + L::A.res + 32 * j) / 16),
                        dsc(kDescSw128, st4 + (kW + L::W.b + 32 * j) / 16), idesc_bs(false, MX, id, id),
                        (t_sfa_res + 4 * atom) | (id << 30), (t_sfb_res + 8 * atom) | (id << 30), accumulate);
          accumulate = 1u;
        }
      }
    }
    tc_commit_both(done);  // arrives in both CTAs once every MMA above has completed
  }
  if (threadIdx.x == 0) {
    volatile uint32_t no_abort = 0;
    mbar_wait(done, 0, limit_ns, &no_abort);  // on expiry the device status records it
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

template <bool MX, int MODE>
cudaError_t launch_peak_t(int iters, int clusters, cudaStream_t st) {
  static std::once_flag once[64];
  static cudaError_t err[64];
  static int sms[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev] {
    err[dev] = cudaFuncSetAttribute(mma_peak_kernel<MX, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kPeakSmemBytes);
    if (err[dev] == cudaSuccess) err[dev] = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
  });
  if (err[dev] != cudaSuccess) return err[dev];
  const int pairs = clusters > 0 && clusters < sms[dev] / 2 ? clusters : sms[dev] / 2;
  // a wait limit far above the loop's length (~0.5 us per K step at the lowest clocks seen)
  const unsigned long long limit = 4000000000ull + 2000ull * (unsigned long long)iters;
  mma_peak_kernel<MX, MODE><<<2 * pairs, kPeakThreads, kPeakSmemBytes, st>>>(iters, limit);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D map over `rows` rows of `inner` elements (uint8 or uint32), box `box_inner` x `box_rows`.
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint64_t inner, uint64_t rows,
              uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t esz = dt == CU_TENSOR_MAP_DATA_TYPE_UINT32 ? 4 : 1;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * esz};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Host-side launch cost matters at these kernel durations (tens of microseconds): tensor
// maps are cached by (base, rows, box) -- a map encodes nothing but the address and shape --
// and the per-device setup (shared-memory opt-in, SM count) is done once per device.
struct MapCache {
  struct Entry {
    const void *base;
    uint64_t rows;
    uint32_t box_rows;
    CUtensorMap map;
  };
  static constexpr int kEntries = 32;
  std::mutex mu;
  Entry e[kEntries];
  int used = 0, next = 0;

  bool get(CUtensorMap *out, const void *base, uint64_t rows, uint32_t box_rows) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
      if (e[i].base == base && e[i].rows == rows && e[i].box_rows == box_rows) {
        *out = e[i].map;
        return true;
      }
    // chunk rows of 1024 bytes (256 x u32), one box = one chunk
    if (!make_map(out, base, CU_TENSOR_MAP_DATA_TYPE_UINT32, 256, rows, 256, box_rows, CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
    Entry &slot = e[used < kEntries ? used++ : next];
    if (used == kEntries) next = (next + 1) % kEntries;
    slot.base = base;
    slot.rows = rows;
    slot.box_rows = box_rows;
    slot.map = *out;
    return true;
  }
};

constexpr int kMaxDevices = 64;

template <bool MX, bool SPARSE, int MAXG, bool PAIR>
cudaError_t launch_t(const TmaMapSet<MAXG> &ms, const GemmParams &p, cudaStream_t st) {
  static std::once_flag once[kMaxDevices];
  static cudaError_t setup_err[kMaxDevices];
  static int sms[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  auto kern = PAIR ? sharq_gemm_kernel<MX, SPARSE, MAXG> : sharq_gemm1_kernel<MX, SPARSE, MAXG>;
  constexpr int smem = PAIR ? kSmemBytes : kSmemBytes1;
  std::call_once(once[dev], [dev, kern] {
    setup_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (setup_err[dev] == cudaSuccess)
      setup_err[dev] = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
  });
  if (setup_err[dev] != cudaSuccess) return setup_err[dev];
  if (p.num_tiles == 0) return cudaSuccess;
  // persistent: one CTA pair per two SMs, or one CTA per SM, at most one per tile
  const int units = PAIR ? sms[dev] / 2 : sms[dev];
  const int grid = (p.num_tiles < units ? p.num_tiles : units) * (PAIR ? 2 : 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may start while the previous kernel drains
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, ms, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Tensor maps of one group: activation and weight chunks (cached), bf16 output.
bool group_maps(TmaMaps *maps, const GemmParams &p, const GemmGroup &G) {
  static MapCache cache;
  const int fmt = p.fmt == kFmtMX ? 1 : 0;
  const ActTile A = act_tile(fmt, 2, p.sparse != 0);
  const WTile W = w_tile(fmt);
  const uint64_t ks = (uint64_t)p.K / BK;
  const uint64_t a_rows = (uint64_t)(G.T_pad / 128) * ks * (A.bytes / 1024);
  const uint64_t w_rows = (uint64_t)(p.N_pad / 128) * ks * (W.bytes / 1024);
  memset(&maps->y, 0, sizeof maps->y);
  if (!p.out_f32 && G.T > 0) {
    auto fn = encode_fn();
    cuuint64_t dims[2] = {(cuuint64_t)p.N, (cuuint64_t)G.T};
    cuuint64_t strides[1] = {(cuuint64_t)p.N * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    if (!fn || fn(&maps->y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, G.y, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  if (G.T == 0) {  // no tiles: the maps are never used
    memset(&maps->act, 0, sizeof maps->act);
    memset(&maps->w, 0, sizeof maps->w);
    return true;
  }
  return cache.get(&maps->act, G.a_tiles, a_rows, A.bytes / 1024) && cache.get(&maps->w, G.w_tiles, w_rows, W.bytes / 1024);
}

template <int MAXG>
cudaError_t launch_groups(const GemmParams &p, cudaStream_t st, const char **why) {
  TmaMapSet<MAXG> ms;
  for (int g = 0; g < p.n_groups; ++g)
    if (!group_maps(&ms.m[g], p, p.grp[g])) {
      *why = "cuTensorMapEncodeTiled failed (driver entry point missing or operand layout rejected)";
      return cudaErrorInvalidValue;
    }
  const bool mx = p.fmt == kFmtMX;
  if (p.sparse && p.single)
    return mx ? launch_t<true, true, MAXG, false>(ms, p, st) : launch_t<false, true, MAXG, false>(ms, p, st);
  if (p.sparse) return mx ? launch_t<true, true, MAXG, true>(ms, p, st) : launch_t<false, true, MAXG, true>(ms, p, st);
  return mx ? launch_t<true, false, MAXG, true>(ms, p, st) : launch_t<false, false, MAXG, true>(ms, p, st);
}

}  // namespace

// Single-CTA tiles (128 rows) against CTA-pair tiles (256 rows) for a sparse launch: the one
// whose rounds of tiles over the persistent grid take less time, a single-CTA tile costing
// 1.1 pair tiles (it moves both weight halves into one SM: measured ~7 % slower at equal
// rounds). A problem of at most 128 rows pads a pair tile by half; the single-CTA form wins
// where that padding adds rounds (a mixture-of-experts layer, a split-K launch), not for a
// lone small launch that fits in one round either way.
bool use_single_cta(const GemmParams &p) {
  if (!p.sparse) return false;
  const int sms = sm_count();
  if (sms < 2) return false;
  const long long num_n = (p.N + BN - 1) / BN;
  long long pair_tiles = 0, single_tiles = 0;
  for (int g = 0; g < p.n_groups; ++g) {
    pair_tiles += (p.grp[g].T + 2 * BM - 1) / (2 * BM) * num_n;
    single_tiles += (p.grp[g].T + BM - 1) / BM * num_n;
  }
  const long long pair_rounds = (pair_tiles + sms / 2 - 1) / (sms / 2);
  const long long single_rounds = (single_tiles + sms - 1) / sms;
  return 10 * pair_rounds > 11 * single_rounds;
}

// Fills the tile ranges of p.grp[0 .. n_groups) and launches one kernel.
cudaError_t launch_gemm(GemmParams p, cudaStream_t st, const char **why) {
  int tiles = 0;
  const int num_n = (p.N + BN - 1) / BN;
  p.single = use_single_cta(p) ? 1 : 0;
  const int rows_per_tile = p.single ? BM : 2 * BM;
  for (int g = 0; g < p.n_groups; ++g) {
    if (p.grp[g].num_k == 0) p.grp[g].num_k = p.K / BK - p.grp[g].k0;
    p.grp[g].num_m = (p.grp[g].T + rows_per_tile - 1) / rows_per_tile;
    p.grp[g].tile_begin = tiles;
    tiles += p.grp[g].num_m * num_n;
  }
  p.num_tiles = tiles;
  return p.n_groups == 1 ? launch_groups<1>(p, st, why) : launch_groups<kMaxGroups>(p, st, why);
}

// ---------------------------------------------------------------- split K
// A launch with few output tiles leaves most SM pairs idle; its K range is then cut into S
// slices, run as S groups of one grouped launch that write float32 partial outputs (each
// already scaled by s_x * s_w), and summed in slice order by a second kernel.
int sm_count() {
  static std::once_flag once[kMaxDevices];
  static int sms[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::call_once(once[dev], [dev] {
    if (cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms[dev] = 0;
  });
  return sms[dev];
}

// Slices for a (tokens x n_out x k) linear, from a cost estimate: a pair (or, for at most 128
// rows, a single CTA) spends about 0.5 us per K step of a tile (the tensor pipe's rate at these
// tile sizes), so one slice of q steps saves (K steps - q) * 0.5 us when every unit holds at
// most one tile; the split form costs a
// second launch (~3 us) and the float32 partials written and read back (S * tokens * n_out *
// 8 bytes at ~3 TB/s, L2-resident). 1 when the tiles already fill half of the SM pairs or
// slicing does not pay; at most kMaxGroups slices, at least 2 K steps each.
int gemm_split_count(int tokens, int n_out, int k) {
  // at most 128 rows: the single-CTA form (one 128-row tile per SM), else CTA pairs
  const bool single = tokens <= BM;
  const int pairs = single ? sm_count() : sm_count() / 2;
  const int rows = single ? BM : 2 * BM;
  const int tiles = ((tokens + rows - 1) / rows) * ((n_out + BN - 1) / BN);
  const int ks = k / BK;
  if (pairs < 2 || 2 * tiles > pairs) return 1;
  int s_max = pairs / tiles;
  if (s_max > kMaxGroups) s_max = kMaxGroups;
  if (s_max > ks / 2) s_max = ks / 2;
  double best = 0.5 * ks;
  int best_s = 1;
  for (int S = 2; S <= s_max; ++S) {
    const int q = (ks + S - 1) / S;
    const double est = 0.5 * q + 3.0 + (double)S * tokens * n_out * 8.0 / 3.0e6;
    if (est < best) {
      best = est;
      best_s = (ks + q - 1) / q;  // every slice non-empty
    }
  }
  return best_s;
}

namespace {
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float4 *ws, int S, long long n4, long long plane4,
                                                            void *y, int out_f32) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float4 a = __ldcs(ws + i);
    for (int s = 1; s < S; ++s) {  // slice order: a fixed summation order
      const float4 b = __ldcs(ws + s * plane4 + i);
      a.x = __fadd_rn(a.x, b.x);
      a.y = __fadd_rn(a.y, b.y);
      a.z = __fadd_rn(a.z, b.z);
      a.w = __fadd_rn(a.w, b.w);
    }
    if (out_f32) {
      reinterpret_cast<float4 *>(y)[i] = a;
    } else {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
      reinterpret_cast<uint2 *>(y)[i] =
          make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
    }
  }
}
}  // namespace

cudaError_t launch_splitk_reduce(const float *ws, int S, int T, int N, void *y, int out_f32, cudaStream_t st) {
  const long long n4 = (long long)T * N / 4;  // N is a multiple of 16
  long long blocks = (n4 + 255) / 256;
  const long long cap = 8ll * (sm_count() > 0 ? sm_count() : 148);
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  splitk_reduce_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const float4 *>(ws), S, n4, n4, y, out_f32);
  return cudaGetLastError();
}

cudaError_t launch_mma_peak(int mode, int fmt, int iters, int clusters, cudaStream_t st) {
  const bool mx = fmt == kFmtMX;
  if (mode == 0) return mx ? launch_peak_t<true, 0>(iters, clusters, st) : launch_peak_t<false, 0>(iters, clusters, st);
  if (mode == 1) return mx ? launch_peak_t<true, 1>(iters, clusters, st) : launch_peak_t<false, 1>(iters, clusters, st);
  return mx ? launch_peak_t<true, 2>(iters, clusters, st) : launch_peak_t<false, 2>(iters, clusters, st);
}

cudaError_t read_and_clear_device_status(int *status, cudaStream_t st) {
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  uint32_t v = 0, zero = 0;
  if ((e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof v)) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero)) != cudaSuccess) return e;
  *status = (int)v;
  return cudaSuccess;
}

}  // namespace sharq
