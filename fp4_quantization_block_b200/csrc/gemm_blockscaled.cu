// gemm_blockscaled.cu -- block-scaled FP4 GEMM on the sm_100a tensor cores.
//
//   D[m][n] = alpha * sum_k A[m][k] * B[n][k]
//
// A and B are FP4 operands as the quantizers emit them: packed E2M1 payload
// (K-major, two values per byte) plus one scale byte per block in 128x4
// atoms ("FP4 Is No Longer Just a Hardware Feature -- The NVFP4 Software
// Stack Is Taking Shape", section "NVFP4 is more than a 4-bit value": the
// contract is payload + block scales + tensor scale + a defined layout; the
// GEMM is the consumer whose layout the producer matches, "Format-Aware
// Fusion: The Engineering Practice That Doubles FP4 Pretraining Throughput",
// section "The Design Philosophy of Format-Aware Fusion").
//
// The kernel (gemm_st::gemm_st_kernel, below): scale factors staged into
// tensor memory by tcgen05.st from their own pipeline, 1-SM or 2-SM
// (cta_group::2) tiles, output through shared memory and bulk-tensor
// stores, optionally the output's MXFP4 operand from the epilogue.
// NVFP4-CTA-local: the second-level scale differs per 128-wide K chunk, so
// each chunk accumulates into one of two tensor-memory partials (the MMAs
// may run one chunk ahead) that the epilogue warps fold,
// tsA[m/128][kc] * tsB[n/128][kc] * partial, into FP32 registers as soon as
// the chunk's MMAs complete; 128-wide 1-SM tiles (a 2-SM 256 x 128 pair
// form is kept in the template but not dispatched: measured slower).
//
// Ragged shapes (M, N any; K a multiple of 32): the grid covers whole tiles;
// TMA reads zeros for payload outside A and B, scale atoms that the operands
// do not have (past the last 128-row block, or past the last atom along K)
// are staged as zero bytes, and the stores skip what lies outside D.  Zero
// payload times a finite scale adds nothing, so the padded tile computes
// the exact result of the smaller one.
//
// Every mbarrier wait is bounded: past `timeout_ns` the waiting thread sets
// the device status word, raises a CTA-wide abort flag and leaves its loop;
// the CTA then waits (bounded) for its own copies in flight, frees its
// tensor memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <cuda_bf16.h>

#include "fa4_device.cuh"
#include "fa4_kernels.h"
#include "launch.cuh"

namespace fa4 {
namespace gemm {

constexpr int BM = 128;
constexpr int BK = 256;            // elements per k-tile (128 bytes per row)
constexpr int BKB = BK / 2;        // bytes per row per k-tile
constexpr int TMEM_COLS = 512;
constexpr uint32_t kStatusTimeout = 7;

// ------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// One bounded probe of a barrier phase.  With HINT, a suspend-time hint
// (1 ms) lets the hardware park the waiting warp until the phase completes
// instead of returning at once, so waiting warps take no issue slots from
// the working ones: measured 4-5% faster for the MXFP4 / NVFP4-global GEMM,
// 6% slower for the CTA-local one, whose fold warps wait on a short chunk
// hand-off.  Callers still loop on it against their own time limit.
template <bool HINT = true>
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  if constexpr (HINT)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 1000000;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
  return ok != 0;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
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
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
template <int KIND>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  if constexpr (KIND == kMX) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
  }
}
// 32 lanes x 32 consecutive 32-bit columns -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (sm_100 layout): start address >> 4 in
// bits 0-13, leading byte offset >> 4 in 16-29, stride byte offset >> 4 in
// 32-45, version 1 in bits 46-47, layout type in 61-63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(sbo >> 4) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
// K-major operand tile, rows of 128 bytes, 128-byte swizzle, 8-row groups
// 1024 bytes apart.
__device__ __forceinline__ uint64_t operand_desc(uint32_t addr) {
  return smem_desc(addr, 16, 1024, 2);
}
// Block-scaled instruction descriptor: E2M1 A and B (format 1), K-major,
// N >> 3 in bits 17-22, scale type in bit 23 (1 = E8M0, 0 = E4M3), M >> 4
// in bits 24-28, scale-factor byte ids in bits 4-5 (B) and 29-30 (A).
template <int KIND, int N>
__device__ __forceinline__ uint32_t instr_desc(uint32_t sf_id) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((KIND == kMX ? 1u : 0u) << 23) | ((uint32_t)(BM >> 4) << 24) | (sf_id << 4) |
         (sf_id << 29);
}

template <int KIND>
struct Cfg {  // KIND kMX: 32-blocks; kNVG / kNVC: 16-blocks
  static constexpr int BS = (KIND == kMX) ? 32 : 16;   // block size
  static constexpr int SF_PER_ROW = BK / BS;           // scale bytes per row per k-tile
  static constexpr int ATOMS_K = SF_PER_ROW / 4;       // 128x4 atoms along K per k-tile
  static constexpr int SFA_BYTES = ATOMS_K * 512;      // per 128 rows
};

struct Params {
  const uint8_t *a_scales, *b_scales;
  const float *a_ts, *b_ts;
  int64_t M, N, K;
  float alpha;
  void *D;
  int64_t ldd;
  int out_fp32;
  uint32_t *status;
  int debug_skip_stage;
  uint64_t timeout_ns;
  int n_fastest;  // tile order: 1 = walk N first (B stays in L2), 0 = walk M first
  // epilogue quantization of the bf16 output to its row-wise MXFP4 operand
  // (payload [M, N/2], scales in the 128x4 atom layout); null: none
  uint8_t *q_payload, *q_scales;
  int store_d;  // 0: D is not written (only the quantized operand)
  // ragged shapes: some tile reaches past M, N or K (see the file comment)
  int ragged;
  int64_t rb_a, rb_b;  // 128-row blocks of A and B (atom rows of their scales)
};

// Output tile coordinates of linear tile index t.  Concurrently running CTAs
// take consecutive t, so the operand along the fast dimension is re-read by
// every row (column) of tiles and should be the one that fits in L2.
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int n_fastest, int &mt,
                                            int &nt) {
  if (n_fastest) {
    mt = t / num_n;
    nt = t % num_n;
  } else {
    mt = t % num_m;
    nt = t / num_m;
  }
}

}  // namespace gemm

// ==========================================================================
// PTX helpers for 2-SM (cta_group::2) tiles.  A cluster of two CTAs (ranks 0
// and 1) computes a 256 x 256 output tile with tcgen05.mma.cta_group::2
// (M = 256, N = 256): CTA r holds A rows 128r..128r+127 and B rows
// 128r..128r+127 of the pair tile in its shared memory and receives D rows
// 128r..128r+127 (all 256 columns) in its tensor memory, so each SM moves
// half the B operand of a 1-SM tile for the same MMA work.  Both CTAs' TMA
// loads complete on the leader's barrier; the leader's commits arrive on
// the barriers of both CTAs (commit multicast).  No TMA load uses cluster
// multicast.
// ==========================================================================
namespace gemm2 {

using namespace fa4::gemm;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared variable in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// TMA tile load into this CTA's shared memory whose completion is counted on
// a barrier of either CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}
// commit of the pair's MMAs: arrive on the barrier at this offset in every
// CTA of `mask`
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          bar),
      "h"(mask)
      : "memory");
}
template <int KIND>
__device__ __forceinline__ void tc_mma_pair(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  if constexpr (KIND == kMX) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
  }
}
// instruction descriptor for the pair: M = 256, N = 256 (or 128: the
// CTA-local form, whose chunk partials must leave room in tensor memory)
template <int KIND, int N = 256>
__device__ __forceinline__ uint32_t instr_desc_pair(uint32_t sf_id) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((KIND == kMX ? 1u : 0u) << 23) |
         ((uint32_t)(256 >> 4) << 24) | (sf_id << 4) | (sf_id << 29);
}

}  // namespace gemm2

// ==========================================================================
// Scale staging by tcgen05.st with a separate scale pipeline.
//
// Output tiles of 128 x BN per CTA (PAIR = false) or 256 x 256 per cluster
// pair with tcgen05.mma.cta_group::2 (PAIR = true, see gemm2), persistent.
// The scale factors take their own path to tensor memory:
//   warp 10      scale producer: per k-tile, the A and B scale atoms
//                (contiguous 512-byte runs) by cp.async.bulk into a deep
//                ring of small shared-memory stages (SF_STAGES);
//   warps 2..9   scale staging + epilogue, two warps per 32-lane quadrant
//                taking alternate k-tiles: a warp reads its k-tile's atoms
//                from shared memory and writes, with tcgen05.st, the words
//                its quadrant's MMA slice reads (row 32q + l of A in column
//                4a + q; all B rows of atom a in columns (BN/32)a ..) into a
//                ring of NBUF tensor-memory buffers, up to NBUF k-tiles ahead
//                of the MMA; at the end of each tile each warp reads half of
//                its quadrant's accumulator columns, releases the
//                accumulator, and writes 32 rows x 64 bytes at a time into a
//                private shared-memory buffer that a bulk-tensor store copies
//                to D (with QOUT it also quantizes each 32-column MXFP4 block
//                of its rows);
//   warp 0       A/B producer: two TMA tile loads per k-tile (AB_STAGES);
//   warp 1       MMA issue (the pair's leader only).
// Neither tcgen05.cp (whose per-instruction cost in the tensor pipe rivals
// an MMA) nor the scale staging sits between an A/B stage landing and its
// MMAs, and the A/B producer issues only two copies per k-tile.  In a pair
// each CTA stages its own A rows' scales and all 256 B rows' scales into its
// own tensor memory; the leader's MMA waits for both CTAs' stagers.
// ==========================================================================
namespace gemm_st {

using namespace fa4::gemm;
using namespace fa4::gemm2;

constexpr int NBUF = 5;       // scale buffers in tensor memory (at most)
constexpr int SF_BASE = 256;  // first column after a 256-column accumulator
constexpr int NUM_THREADS_ST = 352;  // 11 warps

template <int KIND, int BN, bool PAIR>
struct CfgSt {
  using C = Cfg<KIND>;
  static constexpr int TILE_M = PAIR ? 256 : 128;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;            // B rows in this CTA
  static constexpr int A_BYTES = 128 * BKB;
  static constexpr int B_BYTES = B_ROWS * BKB;
  static constexpr int SFA_BYTES = C::SFA_BYTES;                // 128 rows
  static constexpr int SFB_BYTES = C::SFA_BYTES * (BN / 128);   // all BN rows
  static constexpr int AB_BYTES = A_BYTES + B_BYTES;
  static constexpr int SF_BYTES = SFA_BYTES + SFB_BYTES;
  static constexpr int SF_STAGES = BN == 256 ? 5 : 8;
  // epilogue staging: EPI_BUFS buffers of one 32-row x 64-byte output chunk
  // per epilogue warp (a warp fills one while the bulk-tensor engine reads
  // the other)
  static constexpr int EPI_BUFS = 2;
  static constexpr int EPI_WARP_BYTES = 2048 * EPI_BUFS;
  static constexpr int EPI_BYTES = 8 * EPI_WARP_BYTES;
  static constexpr int SMEM_LIMIT = 232448;  // 227 KB per block (opt-in)
  static constexpr int RESERVE = 2048;       // control block + alignment slack
  static constexpr int BUDGET = SMEM_LIMIT - RESERVE - EPI_BYTES;
  static constexpr int AB_STAGES_RAW = (BUDGET - SF_STAGES * SF_BYTES) / AB_BYTES;
  static constexpr int AB_STAGES = AB_STAGES_RAW > 6 ? 6 : AB_STAGES_RAW;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + AB_STAGES * A_BYTES;
  static constexpr int OFF_SF = OFF_B + AB_STAGES * B_BYTES;
  static constexpr int OFF_EPI = OFF_SF + SF_STAGES * SF_BYTES;
  static constexpr int OFF_CTRL = OFF_EPI + EPI_BYTES;
  static_assert(OFF_EPI % 1024 == 0, "64-byte swizzle needs 512-byte aligned chunks");
  // tensor-memory columns of one scale buffer
  static constexpr int COLS_A = C::ATOMS_K * 4;
  static constexpr int COLS_B = C::ATOMS_K * (BN / 32);
  static constexpr int COLS_BUF = COLS_A + COLS_B;
  // CTA-local NVFP4 keeps two 128-column chunk partials (the MMA may run one
  // chunk ahead of the fold) and five scale buffers after them, like the
  // other formats' one accumulator and five scale buffers (a third partial,
  // at the cost of a scale buffer, measured 6-10% slower)
  static constexpr int NPART = 2;
  static constexpr int SF_COL0 = KIND == kNVC ? NPART * 128 : SF_BASE;
  static constexpr int NBUF_ST = NBUF;
  // warps arriving per k-tile on a scale buffer (one per lane quadrant, in
  // each CTA of a pair) and per tile on the accumulator (two per quadrant)
  static constexpr int SF_ARRIVALS = PAIR ? 8 : 4;
  static constexpr int ACC_ARRIVALS = PAIR ? 16 : 8;
  static_assert(!PAIR || BN == 256 || (KIND == kNVC && BN == 128),
                "a pair computes 256-wide tiles (CTA-local NVFP4: 128-wide)");
  static_assert(AB_STAGES >= 2, "shared-memory budget");
  static_assert(SF_COL0 + NBUF_ST * COLS_BUF <= TMEM_COLS, "tensor-memory budget");
  static_assert(NBUF_ST <= NBUF, "barrier arrays");
};

struct SmemSt {
  uint64_t ab_full[6], ab_empty[6];
  uint64_t sfs_full[12], sfs_empty[12];      // scale stages in shared memory
  uint64_t sft_full[NBUF], sft_empty[NBUF];  // scale buffers in tensor memory
  uint64_t acc_full, acc_empty, mma_done;
  uint64_t part_full[3], part_empty[3];  // CTA-local NVFP4: the 128-K chunk partials
  uint32_t tmem_base;
  int abort;
};

template <int KIND, int BN, bool PAIR>
constexpr int total_smem_st() {
  static_assert(CfgSt<KIND, BN, PAIR>::OFF_CTRL + (int)sizeof(SmemSt) + 1024 <=
                    CfgSt<KIND, BN, PAIR>::SMEM_LIMIT,
                "shared-memory limit");
  return CfgSt<KIND, BN, PAIR>::OFF_CTRL + (int)sizeof(SmemSt) + 1024;
}

template <bool HINT>
__device__ __forceinline__ bool wait_st(uint32_t bar, uint32_t parity, SmemSt *sm, const Params &p,
                                        uint32_t where) {
  if (mbar_try_wait<HINT>(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait<HINT>(bar, parity)) return true;
    if (*(volatile int *)&sm->abort) return false;
    if (globaltimer() - t0 > p.timeout_ns) {
      *(volatile int *)&sm->abort = 1;
      if (atomicCAS(p.status, 0u, kStatusTimeout) == 0u) atomicExch(p.status + 1, where);
      return false;
    }
  }
}
// every lane of the warp probes the barrier; the vote keeps the outcome
// uniform even if a lane's wait ran out while another's phase completed
template <bool HINT>
__device__ __forceinline__ bool warp_wait_st(uint32_t bar, uint32_t parity, SmemSt *sm,
                                             const Params &p, uint32_t where) {
  return __all_sync(0xFFFFFFFFu, wait_st<HINT>(bar, parity, sm, p, where));
}
// wait until the last copy issued into each stage of a ring has landed
__device__ __forceinline__ void drain_ring(uint64_t *full, int n, uint32_t issued,
                                           uint32_t last_parity, const Params &p, uint32_t where) {
  for (int s = 0; s < n; ++s) {
    if (!((issued >> s) & 1u)) continue;
    const uint32_t par = (last_parity >> s) & 1u;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(smem_u32(&full[s]), par)) {
      if (globaltimer() - t0 > p.timeout_ns) {
        if (atomicCAS(p.status, 0u, kStatusTimeout) == 0u) atomicExch(p.status + 1, where | s);
        break;
      }
    }
  }
}

// Arrive on a barrier of the pair's leader from the peer CTA.  Relaxed: what
// the arrival publishes is tensor memory already completed by
// tcgen05.wait::st / wait::ld and ordered by tcgen05.fence, and a release at
// cluster scope would also wait for this thread's outstanding global stores
// (measured ~1000 cycles per arrival).
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

// Output tile store through shared memory: the bulk-tensor (TMA) engine
// writes whole lines, so the epilogue issues no per-row global stores.
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// The stores carry an L2 evict-first policy: the output streams out to DRAM
// while the GEMM computes, instead of lingering dirty in L2 and being
// written back during whatever memory-bound kernel runs next.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y,
                                             uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%1, %2}], [%3], %4;" ::"l"(map),
      "r"(x), "r"(y), "r"(src), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the shared-memory source of all but the N most recent committed stores
// has been read
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// every committed store has completed
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint4 &v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// N consecutive columns (N = 8, 16 or 32) of this warp's 32 lanes, one
// word per lane and column
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t *v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t *v) {
  static_assert(N == 8 || N == 16 || N == 32, "column count");
  if constexpr (N == 8) {
    tmem_st8(taddr, v);
  } else {
    tmem_st16(taddr, v);
    if constexpr (N == 32) tmem_st16(taddr + 16, v + 16);
  }
}

// RAG: some tile reaches past M, N or K (Params::ragged); aligned shapes run
// an instantiation without the edge checks
template <int KIND, int BN, bool PAIR, bool QOUT, bool RAG>
__global__ void __launch_bounds__(NUM_THREADS_ST, 1)
    gemm_st_kernel(const __grid_constant__ CUtensorMap map_a,
                   const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_d, const Params p) {
  using CS = CfgSt<KIND, BN, PAIR>;
  constexpr bool kHint = KIND != kNVC;  // see mbar_try_wait
  using C = Cfg<KIND>;
  constexpr int ABS = CS::AB_STAGES, SFS = CS::SF_STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  SmemSt *sm = reinterpret_cast<SmemSt *>(smem + CS::OFF_CTRL);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;      // tile-walking unit
  const int nunits = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  const int num_m = (int)((p.M + CS::TILE_M - 1) / CS::TILE_M);
  const int num_n = (int)((p.N + BN - 1) / BN);
  const int num_tiles = num_m * num_n;
  const int KT = (int)((p.K + BK - 1) / BK);
  const int64_t kbt4 = (p.K / C::BS + 3) / 4;  // atoms along K per 128-row block
  const int my_tiles = unit < num_tiles ? (num_tiles - unit + nunits - 1) / nunits : 0;
  const int total = my_tiles * KT;  // k-tiles this CTA processes

  if (threadIdx.x == 0) {
    for (int s = 0; s < ABS; ++s) {
      mbar_init(smem_u32(&sm->ab_full[s]), 1);
      mbar_init(smem_u32(&sm->ab_empty[s]), 1);
    }
    for (int s = 0; s < SFS; ++s) {
      mbar_init(smem_u32(&sm->sfs_full[s]), 1);
      mbar_init(smem_u32(&sm->sfs_empty[s]), 4);
    }
    for (int b = 0; b < CS::NBUF_ST; ++b) {
      mbar_init(smem_u32(&sm->sft_full[b]), CS::SF_ARRIVALS);
      mbar_init(smem_u32(&sm->sft_empty[b]), 1);
    }
    mbar_init(smem_u32(&sm->acc_full), 1);
    mbar_init(smem_u32(&sm->acc_empty), CS::ACC_ARRIVALS);
    for (int c = 0; c < CS::NPART; ++c) {
      mbar_init(smem_u32(&sm->part_full[c]), 1);
      mbar_init(smem_u32(&sm->part_empty[c]), CS::ACC_ARRIVALS);
    }
    mbar_init(smem_u32(&sm->mma_done), 1);
    sm->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&sm->tmem_base)),
                   "r"(TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&sm->tmem_base)),
                   "r"(TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {
    __syncwarp();
    cluster_sync();  // the peer's barriers exist before any remote arrive
  }
  tc_fence_after();
  // the prologue above touches no global memory; the previous kernel in the
  // stream may still be running until here
  grid_dependency_wait();
  grid_dependents_launch();
  const uint32_t tmem = sm->tmem_base;
  // barriers the pair's MMA waits on live in the leader (rank 0)
  auto leader_addr = [&](const void *local) -> uint32_t {
    return PAIR ? map_to_rank(smem_u32(local), 0) : smem_u32(local);
  };

  if (warp == 0) {
    // ------------------------------------------------------ A/B producer
    if (lane == 0) {
      uint32_t issued = 0, last_parity = 0;
      int g = 0;
      bool ok = true;
      for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
        int mt, nt;
        tile_coords(tile, num_m, num_n, p.n_fastest, mt, nt);
        for (int kt = 0; kt < KT; ++kt, ++g) {
          const int s = g % ABS;
          const uint32_t ph = (uint32_t)((g / ABS) & 1);
          if (!wait_st<kHint>(smem_u32(&sm->ab_empty[s]), ph ^ 1u, sm, p, 0x100u | s)) {
            ok = false;
            break;
          }
          if (g == p.debug_skip_stage) continue;
          const uint32_t a_dst = smem_u32(smem + CS::OFF_A + s * CS::A_BYTES);
          const uint32_t b_dst = smem_u32(smem + CS::OFF_B + s * CS::B_BYTES);
          if constexpr (PAIR) {
            const uint32_t fb = leader_addr(&sm->ab_full[s]);
            if (rank == 0) mbar_arrive_expect_tx(smem_u32(&sm->ab_full[s]), 2 * CS::AB_BYTES);
            tma_load_2d_pair(a_dst, &map_a, kt * BKB, mt * 256 + (int)rank * 128, fb);
            tma_load_2d_pair(b_dst, &map_b, kt * BKB, nt * BN + (int)rank * (BN / 2), fb);
          } else {
            const uint32_t fb = smem_u32(&sm->ab_full[s]);
            mbar_arrive_expect_tx(fb, CS::AB_BYTES);
            tma_load_2d(a_dst, &map_a, kt * BKB, mt * BM, fb);
            tma_load_2d(b_dst, &map_b, kt * BKB, nt * BN, fb);
          }
          issued |= 1u << s;
          last_parity = (last_parity & ~(1u << s)) | (ph << s);
        }
      }
      if (!PAIR || rank == 0) {
        drain_ring(sm->ab_full, ABS, issued, last_parity, p, 0x400u);
      } else if (!ok) {
        // the peer's copies complete on the leader's barriers: give any
        // copy still in flight time to land before this CTA can leave
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 10) {
    // --------------------------------------------------- scale producer
    if (lane == 0) {
      uint32_t issued = 0, last_parity = 0;
      int g = 0;
      bool ok = true;
      for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
        int mt, nt;
        tile_coords(tile, num_m, num_n, p.n_fastest, mt, nt);
        const int rb_a = PAIR ? mt * 2 + (int)rank : mt;
        for (int kt = 0; kt < KT; ++kt, ++g) {
          const int s = g % SFS;
          const uint32_t ph = (uint32_t)((g / SFS) & 1);
          if (!wait_st<kHint>(smem_u32(&sm->sfs_empty[s]), ph ^ 1u, sm, p, 0x120u | s)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sm->sfs_full[s]);
          const uint32_t dst = smem_u32(smem + CS::OFF_SF + s * CS::SF_BYTES);
          if (!RAG) {
            mbar_arrive_expect_tx(fb, CS::SF_BYTES);
            bulk_load(dst, p.a_scales + ((int64_t)rb_a * kbt4 + (int64_t)kt * C::ATOMS_K) * 512,
                      CS::SFA_BYTES, fb);
#pragma unroll
            for (int nb = 0; nb < BN / 128; ++nb)
              bulk_load(dst + CS::SFA_BYTES + nb * C::SFA_BYTES,
                        p.b_scales + ((int64_t)(nt * (BN / 128) + nb) * kbt4 + (int64_t)kt * C::ATOMS_K) * 512,
                        C::SFA_BYTES, fb);
          } else {
            // only the atoms the operands have: na along K, and no 128-row
            // block past the last one (at least B's first block exists)
            const int64_t left = kbt4 - (int64_t)kt * C::ATOMS_K;
            const uint32_t bytes = (uint32_t)(left < C::ATOMS_K ? left : C::ATOMS_K) * 512u;
            const bool a_in = rb_a < p.rb_a;
            uint32_t total_bytes = a_in ? bytes : 0u;
#pragma unroll
            for (int nb = 0; nb < BN / 128; ++nb)
              if (nt * (BN / 128) + nb < p.rb_b) total_bytes += bytes;
            mbar_arrive_expect_tx(fb, total_bytes);
            if (a_in)
              bulk_load(dst, p.a_scales + ((int64_t)rb_a * kbt4 + (int64_t)kt * C::ATOMS_K) * 512,
                        bytes, fb);
#pragma unroll
            for (int nb = 0; nb < BN / 128; ++nb)
              if (nt * (BN / 128) + nb < p.rb_b)
                bulk_load(dst + CS::SFA_BYTES + nb * C::SFA_BYTES,
                          p.b_scales + ((int64_t)(nt * (BN / 128) + nb) * kbt4 + (int64_t)kt * C::ATOMS_K) * 512,
                          bytes, fb);
          }
          issued |= 1u << s;
          last_parity = (last_parity & ~(1u << s)) | (ph << s);
        }
      }
      drain_ring(sm->sfs_full, SFS, issued, last_parity, p, 0x420u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issue (leader)
    if (lane == 0 && rank == 0) {
      uint32_t acc_phase = 0;
      bool ok = true;
      int g = 0;
      const uint64_t a_desc0 = operand_desc(smem_u32(smem + CS::OFF_A));
      const uint64_t b_desc0 = operand_desc(smem_u32(smem + CS::OFF_B));
      for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
        if constexpr (KIND != kNVC) {
          if (!wait_st<kHint>(smem_u32(&sm->acc_empty), acc_phase ^ 1u, sm, p, 0x200u)) break;
          tc_fence_after();
        }
        for (int kt = 0; kt < KT; ++kt, ++g) {
          const int s = g % ABS, b = g % CS::NBUF_ST;
          if (!wait_st<kHint>(smem_u32(&sm->sft_full[b]), (uint32_t)((g / CS::NBUF_ST) & 1), sm, p, 0x230u | b) ||
              !wait_st<kHint>(smem_u32(&sm->ab_full[s]), (uint32_t)((g / ABS) & 1), sm, p, 0x210u | s)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // operand descriptors of the stage's first K step: the start
          // address field (address / 16, 14 bits, shared memory stays below
          // 256 KB) advances by 2 per 32-byte K step
          const uint64_t a_desc = a_desc0 + (uint64_t)((s * CS::A_BYTES) >> 4);
          const uint64_t b_desc = b_desc0 + (uint64_t)((s * CS::B_BYTES) >> 4);
          const uint32_t sf_col = tmem + CS::SF_COL0 + b * CS::COLS_BUF;
#pragma unroll
          for (int j = 0; j < BK / 64; ++j) {
            const int a = (KIND == kMX) ? (j >> 1) : j;
            const uint32_t sf_id = (KIND == kMX) ? (uint32_t)(2 * (j & 1)) : 0u;
            const uint32_t sfa = (sf_col + 4 * a) | (sf_id << 30);
            const uint32_t sfb = (sf_col + CS::COLS_A + (BN / 32) * a) | (sf_id << 30);
            if constexpr (KIND == kNVC) {
              // chunk q = 2g + c (MMAs 2c, 2c+1 of this k-tile) starts a
              // fresh partial in buffer q % 3 once the fold has read that
              // buffer's previous chunk
              const int q = 2 * g + (j >> 1), pb = q % CS::NPART;
              if ((j & 1) == 0) {
                if (!wait_st<kHint>(smem_u32(&sm->part_empty[pb]), (uint32_t)(((q / CS::NPART) & 1) ^ 1), sm,
                             p, 0x240u | pb)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
              }
              if constexpr (PAIR)
                tc_mma_pair<KIND>(tmem + 128 * pb, a_desc + 2 * j,
                                  b_desc + 2 * j, instr_desc_pair<KIND, BN>(sf_id),
                                  sfa, sfb, (uint32_t)(j & 1));
              else
                tc_mma<KIND>(tmem + 128 * pb, a_desc + 2 * j,
                             b_desc + 2 * j, instr_desc<KIND, BN>(sf_id), sfa, sfb,
                             (uint32_t)(j & 1));
              if (j & 1) {
                if constexpr (PAIR)
                  tc_commit_pair(smem_u32(&sm->part_full[pb]), (uint16_t)3);
                else
                  tc_commit(smem_u32(&sm->part_full[pb]));
              }
            } else {
              const uint32_t acc = (kt > 0 || j > 0) ? 1u : 0u;
              if constexpr (PAIR)
                tc_mma_pair<KIND>(tmem, a_desc + 2 * j, b_desc + 2 * j,
                                  instr_desc_pair<KIND>(sf_id), sfa, sfb, acc);
              else
                tc_mma<KIND>(tmem, a_desc + 2 * j, b_desc + 2 * j,
                             instr_desc<KIND, BN>(sf_id), sfa, sfb, acc);
            }
          }
          if (!ok) break;
          if constexpr (PAIR) {
            tc_commit_pair(smem_u32(&sm->ab_empty[s]), (uint16_t)3);
            tc_commit_pair(smem_u32(&sm->sft_empty[b]), (uint16_t)3);
          } else {
            tc_commit(smem_u32(&sm->ab_empty[s]));
            tc_commit(smem_u32(&sm->sft_empty[b]));
          }
        }
        if (ok && KIND != kNVC) {
          if constexpr (PAIR)
            tc_commit_pair(smem_u32(&sm->acc_full), (uint16_t)3);
          else
            tc_commit(smem_u32(&sm->acc_full));
        }
        acc_phase ^= 1u;
      }
      if constexpr (PAIR)
        tc_commit_pair(smem_u32(&sm->mma_done), (uint16_t)1);
      else
        tc_commit(smem_u32(&sm->mma_done));
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait<kHint>(smem_u32(&sm->mma_done), 0)) {
        if (globaltimer() - t0 > p.timeout_ns) {
          if (atomicCAS(p.status, 0u, kStatusTimeout) == 0u) atomicExch(p.status + 1, 0x500u);
          break;
        }
      }
    }
  } else {
    // ----------------------------------------- scale staging + epilogue
    const int q = warp & 3;         // tensor-memory lane quadrant of this warp
    const int h = (warp - 2) >> 2;  // which of the quadrant's two warps
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    const uint32_t ebuf = smem_u32(smem + CS::OFF_EPI + (warp - 2) * CS::EPI_WARP_BYTES);
    int epi_next = 0;  // the staging buffer the next output chunk goes through
    constexpr int COLS = BN / 2;
    constexpr int NCH = COLS / 32;
    float alpha_g = p.alpha;
    if constexpr (KIND == kNVG) alpha_g = p.alpha * p.a_ts[0] * p.b_ts[0];
    const uint64_t alpha2 = f2_pack(alpha_g, alpha_g);
    const uint64_t store_policy = l2_evict_first_policy();
    const uint32_t acc_empty_l = leader_addr(&sm->acc_empty);

    // stage the scales of k-tile g into tensor-memory buffer g % NBUF_ST
    auto stage_scales = [&](int g) -> bool {
      const int s = g % SFS, b = g % CS::NBUF_ST;
      if (!warp_wait_st<kHint>(smem_u32(&sm->sfs_full[s]), (uint32_t)((g / SFS) & 1), sm, p, 0x320u | s))
        return false;
      if (g >= CS::NBUF_ST &&
          !warp_wait_st<kHint>(smem_u32(&sm->sft_empty[b]), (uint32_t)(((g / CS::NBUF_ST) & 1) ^ 1), sm, p,
                        0x330u | b))
        return false;
      tc_fence_after();
      const uint8_t *sfa_s = smem + CS::OFF_SF + s * CS::SF_BYTES;
      const uint8_t *sfb_s = sfa_s + CS::SFA_BYTES;
      const uint32_t col = lane_base + CS::SF_COL0 + b * CS::COLS_BUF;
      // ragged shapes: atoms the scale producer did not load are zero
      int na = C::ATOMS_K;
      bool a_in = true, b_in[BN / 128];
#pragma unroll
      for (int nb = 0; nb < BN / 128; ++nb) b_in[nb] = true;
      if (RAG) {
        const int kt = g % KT;
        int mt, nt;
        tile_coords(unit + (g / KT) * nunits, num_m, num_n, p.n_fastest, mt, nt);
        const int64_t left = kbt4 - (int64_t)kt * C::ATOMS_K;
        na = left < C::ATOMS_K ? (int)left : C::ATOMS_K;
        a_in = (PAIR ? mt * 2 + (int)rank : mt) < p.rb_a;
#pragma unroll
        for (int nb = 0; nb < BN / 128; ++nb) b_in[nb] = nt * (BN / 128) + nb < p.rb_b;
      }
      // A: the MMA reads row 32q + lane's word (word q of atom row `lane`) in
      // column 4a + q of this quadrant; the whole atom row goes into columns
      // 4a .. 4a + 3 (the other three words are not read here), so all of
      // the k-tile's A words are COLS_A consecutive columns and one store
      uint32_t aw[CS::COLS_A];
#pragma unroll
      for (int a = 0; a < C::ATOMS_K; ++a) {
        const uint4 v = (a_in && a < na) ? *reinterpret_cast<const uint4 *>(sfa_s + a * 512 + lane * 16)
                                         : make_uint4(0u, 0u, 0u, 0u);
        aw[4 * a] = v.x;
        aw[4 * a + 1] = v.y;
        aw[4 * a + 2] = v.z;
        aw[4 * a + 3] = v.w;
      }
      tmem_st_cols<CS::COLS_A>(col, aw);
      // B: atom a of each 128-row block: row 32w + lane is word w of atom row
      // `lane`, in columns 4 (a * BN/128 + nb) + w: the k-tile's B words are
      // COLS_B consecutive columns, written by one or two wide stores
      constexpr int NBK = BN / 128;
      uint32_t bw[CS::COLS_B];
#pragma unroll
      for (int a = 0; a < C::ATOMS_K; ++a) {
#pragma unroll
        for (int nb = 0; nb < NBK; ++nb) {
          const uint4 v = (b_in[nb] && a < na)
                              ? *reinterpret_cast<const uint4 *>(sfb_s + nb * C::SFA_BYTES + a * 512 + lane * 16)
                              : make_uint4(0u, 0u, 0u, 0u);
          uint32_t *d = &bw[4 * (a * NBK + nb)];
          d[0] = v.x;
          d[1] = v.y;
          d[2] = v.z;
          d[3] = v.w;
        }
      }
      tmem_st_cols<CS::COLS_B>(col + CS::COLS_A, bw);
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&sm->sfs_empty[s]));
        if (PAIR && rank != 0)
          mbar_arrive_remote_relaxed(leader_addr(&sm->sft_full[b]));
        else
          mbar_arrive(smem_u32(&sm->sft_full[b]));
      }
      return true;
    };

    // write one output tile (this warp's 32 rows x COLS columns, accumulator
    // words in r) through the shared-memory buffer and bulk-tensor stores
    auto store_tile = [&](const uint32_t (&r)[COLS], int mt, int nt) {
      // stage 32 rows x 64 bytes at a time in this warp's buffer (16-byte
      // pieces placed with the 64-byte swizzle: piece j of row r at
      // j ^ ((r >> 1) & 3), which the tensor map undoes) and store it with
      // the bulk-tensor engine; the buffer is reused once the previous store
      // has read it
      const int y0 = mt * CS::TILE_M + (int)rank * 128 + 32 * q;
      const int x0 = nt * BN + h * COLS;
      const uint32_t row_off = lane * 64;
      const int sw = (lane >> 1) & 3;
      // ragged shapes: these 32 rows may lie wholly below D (the bulk-tensor
      // store clips a box that only reaches past M or N)
      const bool rows_in = !RAG || (int64_t)y0 < p.M;
      if (p.out_fp32) {
#pragma unroll
        for (int ch = 0; ch < COLS / 16; ++ch) {
          if (RAG && (!rows_in || (int64_t)(x0 + 16 * ch) >= p.N)) continue;
          const uint32_t buf = ebuf + 2048u * (uint32_t)epi_next;
          epi_next = epi_next + 1 == CS::EPI_BUFS ? 0 : epi_next + 1;
          if (lane == 0) bulk_wait_read<CS::EPI_BUFS - 1>();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t *v = &r[16 * ch + 4 * j];
            uint32_t o0, o1, o2, o3;
            f2_unpack_bits(f2_mul(f2_pack_bits(v[0], v[1]), alpha2), o0, o1);
            f2_unpack_bits(f2_mul(f2_pack_bits(v[2], v[3]), alpha2), o2, o3);
            sts128(buf + row_off + 16 * (j ^ sw), o0, o1, o2, o3);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&map_d, buf, x0 + 16 * ch, y0, store_policy);
            bulk_commit();
          }
        }
      } else {
        const int64_t row = (int64_t)y0 + lane;
        uint32_t sword = 0;  // this row's MXFP4 scale bytes, one per 32-column chunk
#pragma unroll
        for (int ch = 0; ch < COLS / 32; ++ch) {
          const bool chunk_in = !RAG || (rows_in && (int64_t)(x0 + 32 * ch) < p.N);
          uint32_t w[16];  // the chunk's 32 bf16 values of D, packed in pairs
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int i = 32 * ch + 2 * u;
            float lo, hi;  // alpha * the pair, one packed multiply (each lane rounded)
            f2_unpack(f2_mul(f2_pack_bits(r[i], r[i + 1]), alpha2), lo, hi);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);
            w[u] = *reinterpret_cast<uint32_t *>(&b2);
          }
          if constexpr (QOUT) {
            // the 32 bf16 values are one MXFP4 block of D's row-wise operand:
            // the same steps as the row-wise quantizer (RNE)
            float f[32];
            float amax = 0.0f;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              f[2 * u] = bf16lo(w[u]);
              f[2 * u + 1] = bf16hi(w[u]);
              amax = fmaxf(amax, fmaxf(fabsf(f[2 * u]), fabsf(f[2 * u + 1])));
            }
            const uint32_t sbyte = mx_scale_byte(amax);
            const float mult = mx_multiplier(sbyte);
#pragma unroll
            for (int e = 0; e < 32; ++e) f[e] = __fmul_rn(f[e], mult);
            const uint4 codes = make_uint4(e2m1x8_rne(&f[0]), e2m1x8_rne(&f[8]),
                                           e2m1x8_rne(&f[16]), e2m1x8_rne(&f[24]));
            // rows and blocks outside D hold zero accumulators: scale byte 0
            if (!RAG || (row < p.M && (int64_t)(x0 + 32 * ch) < p.N))
              *reinterpret_cast<uint4 *>(p.q_payload + row * (p.N >> 1) + ((x0 + 32 * ch) >> 1)) =
                  codes;
            sword |= sbyte << (8 * ch);
          }
          if (p.store_d && chunk_in) {
            const uint32_t buf = ebuf + 2048u * (uint32_t)epi_next;
            epi_next = epi_next + 1 == CS::EPI_BUFS ? 0 : epi_next + 1;
            if (lane == 0) bulk_wait_read<CS::EPI_BUFS - 1>();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j)
              sts128(buf + row_off + 16 * (j ^ sw), w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&map_d, buf, x0 + 32 * ch, y0, store_policy);
              bulk_commit();
            }
          }
        }
        if constexpr (QOUT) {
          // blocks x0/32 .. of this row: a whole scale word (128 columns) or
          // its half (64 columns, the other half is the quadrant's other warp);
          // ragged: rows up to the next multiple of 128 and blocks up to the
          // next multiple of 4 are the operand's padding (written, zero)
          const int64_t nbk = p.N >> 5;
          if (!RAG || (row < p.rb_a * 128 && (int64_t)(x0 >> 5) < nbk)) {
            uint8_t *sdst = p.q_scales + sf_offset(row, x0 >> 5, (nbk + 3) & ~int64_t(3));
            if constexpr (COLS == 128)
              *reinterpret_cast<uint32_t *>(sdst) = sword;
            else
              *reinterpret_cast<uint16_t *>(sdst) = (uint16_t)sword;
          }
        }
      }
    };

    if constexpr (KIND == kNVC) {
      // CTA-local NVFP4: per k-tile, stage this warp's scales up to NBUF_ST
      // k-tiles ahead, then fold the k-tile's two 128-K chunk partials into FP32
      // registers, acc += tsA[m/128][kc] * tsB[n/128][kc] * partial, and
      // release each partial as soon as it is read; store at the tile's end
      const int nk = (int)((p.K + 127) / 128);  // 128-wide K chunks (the last may be short)
      // The chunk factors tsA[mb][kc] * tsB[nt][kc] of this CTA's chunk
      // sequence Q = (tile iteration) * 2 KT + kc, 32 at a time: lane i
      // holds chunk 32 b + i of block b in fcur, the next block in fnext,
      // loaded a whole block (32 chunks of MMAs) before it is needed (a
      // chunk wholly past K, ragged, holds a zero partial and gets factor 0)
      const int cpt = 2 * KT;  // chunks per tile
      auto chunk_factor = [&](int Q) -> float {
        if (Q >= total * 2) return 0.0f;
        const int kc = Q % cpt;
        if (kc >= nk) return 0.0f;
        int mt, nt;
        tile_coords(unit + (Q / cpt) * nunits, num_m, num_n, p.n_fastest, mt, nt);
        const int mb = PAIR ? mt * 2 + (int)rank : mt;  // this CTA's 128-row block of A
        return p.a_ts[(int64_t)mb * nk + kc] * p.b_ts[(int64_t)nt * nk + kc];
      };
      float fcur = chunk_factor(lane), fnext = chunk_factor(32 + lane);
      int g_st = h, g = 0;
      bool ok = true;
      for (int tile = unit; tile < num_tiles && ok; tile += nunits) {
        int mt, nt;
        tile_coords(tile, num_m, num_n, p.n_fastest, mt, nt);
        // (a packed fma.rn.f32x2 fold, same rounding, measured 5% slower:
        // the partial's registers from the tensor-memory load are not
        // paired as its 64-bit operands need)
        float acc[COLS];
#pragma unroll
        for (int i = 0; i < COLS; ++i) acc[i] = 0.0f;
        for (int kt = 0; kt < KT && ok; ++kt, ++g) {
          float fk[2];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int Q = 2 * g + c;
            fk[c] = __shfl_sync(0xFFFFFFFFu, fcur, Q & 31);
            if ((Q & 31) == 31) {
              fcur = fnext;
              fnext = chunk_factor(Q + 33 + lane);
            }
          }
          for (; g_st < total && g_st < g + CS::NBUF_ST; g_st += 2)
            if (!stage_scales(g_st)) {
              ok = false;
              break;
            }
          if (!ok) break;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int q = 2 * g + c, pb = q % CS::NPART;  // chunk q's partial buffer
            if (!warp_wait_st<kHint>(smem_u32(&sm->part_full[pb]), (uint32_t)((q / CS::NPART) & 1), sm, p,
                              0x340u | pb)) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint32_t r[COLS];
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch)
              tmem_ld32(lane_base + 128 * pb + h * COLS + 32 * ch, &r[32 * ch]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (PAIR && rank != 0)
                mbar_arrive_remote_relaxed(leader_addr(&sm->part_empty[pb]));
              else
                mbar_arrive(smem_u32(&sm->part_empty[pb]));
            }
#pragma unroll
            for (int i = 0; i < COLS; ++i) acc[i] = fmaf(fk[c], __uint_as_float(r[i]), acc[i]);
          }
        }
        if (!ok) break;
        uint32_t r[COLS];
#pragma unroll
        for (int i = 0; i < COLS; ++i) r[i] = __float_as_uint(acc[i]);
        store_tile(r, mt, nt);
      }
    } else {
    // the quadrant's two warps stage alternate k-tiles (h = 0 the even ones)
    uint32_t acc_phase = 0;
    int g = h;
    bool ok = true;
    int it = 0;
    for (int tile = unit; tile < num_tiles && ok; tile += nunits, ++it) {
      // scales for the rest of this tile and the first NBUF k-tiles of the
      // next one, then this tile's epilogue
      const int until = min(total, (it + 1) * KT + CS::NBUF_ST);
      for (; g < until; g += 2)
        if (!stage_scales(g)) {
          ok = false;
          break;
        }
      if (!ok) break;
      int mt, nt;
      tile_coords(tile, num_m, num_n, p.n_fastest, mt, nt);
      if (!warp_wait_st<kHint>(smem_u32(&sm->acc_full), acc_phase, sm, p, 0x310u)) break;
      tc_fence_after();
      uint32_t r[COLS];
#pragma unroll
      for (int c = 0; c < NCH; ++c) tmem_ld32(lane_base + h * COLS + 32 * c, &r[32 * c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR && rank != 0)
          mbar_arrive_remote_relaxed(acc_empty_l);
        else
          mbar_arrive(smem_u32(&sm->acc_empty));
      }
      acc_phase ^= 1u;
      store_tile(r, mt, nt);
    }
    }
    // the stores read shared memory and write D after this: both done
    // before the block can leave
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // in a pair neither CTA leaves (or frees tensor memory) while the pair's
  // MMAs may still read its shared memory or write its tensor memory
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {
    __syncwarp();
    cluster_sync();
  }
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    if constexpr (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                   : "memory");
  }
}

}  // namespace gemm_st
}  // namespace fa4

namespace fa4 {

using PFN_encodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                     const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                     const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (a function-local static
// is initialised exactly once even when several host threads call first).
static PFN_encodeTiled get_encode() {
  static const PFN_encodeTiled fn = []() -> PFN_encodeTiled {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_encodeTiled>(ptr);
    return nullptr;
  }();
  return fn;
}

// Payload tile map: uint8 [rows, K/2] row-major, box 128 bytes x box_rows,
// 128-byte swizzle (the layout the MMA's operand descriptors describe).
static bool make_payload_map(CUtensorMap *m, const void *base, int64_t rows, int64_t K,
                             int box_rows) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {(cuuint32_t)gemm::BKB, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_bf16_tile_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map for the bulk-tensor stores: D [M, N] bf16 or fp32 with row
// stride ldd, box 64 bytes x 32 rows, 64-byte swizzle.
static bool make_out_map(CUtensorMap *m, const GemmArgs &a) {
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  const int esz = a.out_fp32 ? 4 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)a.N, (cuuint64_t)a.M};
  cuuint64_t strides[1] = {(cuuint64_t)(a.ldd * esz)};
  cuuint32_t box[2] = {(cuuint32_t)(64 / esz), 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, a.out_fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             a.D, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static gemm::Params make_params(const GemmArgs &a) {
  gemm::Params p;
  p.a_scales = a.a_scales;
  p.b_scales = a.b_scales;
  p.a_ts = a.a_ts;
  p.b_ts = a.b_ts;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.alpha = a.alpha;
  p.D = a.D;
  p.ldd = a.ldd;
  p.out_fp32 = a.out_fp32;
  p.status = a.status;
  p.debug_skip_stage = a.debug_skip_stage;
  p.timeout_ns = a.timeout_ns;
  // keep the smaller operand resident in L2 and stream the larger one once
  p.n_fastest = (a.N <= a.M) ? 1 : 0;
  p.q_payload = a.q_payload;
  p.q_scales = a.q_scales;
  p.store_d = a.D != nullptr;
  p.rb_a = (a.M + 127) / 128;
  p.rb_b = (a.N + 127) / 128;
  p.ragged = 0;  // set by the launcher for its tile shape
  return p;
}

template <int KIND, int BN, bool PAIR, bool QOUT>
static cudaError_t launch_st(const GemmArgs &a, cudaStream_t st) {
  constexpr int smem = gemm_st::total_smem_st<KIND, BN, PAIR>();
  CUtensorMap ma, mb;
  if (!make_payload_map(&ma, a.a_payload, a.M, a.K, gemm::BM)) return cudaErrorInvalidValue;
  if (!make_payload_map(&mb, a.b_payload, a.N, a.K, PAIR ? BN / 2 : BN)) return cudaErrorInvalidValue;
  CUtensorMap md;
  memset(&md, 0, sizeof(md));
  if (a.D && !make_out_map(&md, a)) return cudaErrorInvalidValue;
  gemm::Params p = make_params(a);
  constexpr int TILE_M = PAIR ? 256 : gemm::BM;
  p.ragged = (a.M % TILE_M) || (a.N % BN) || (a.K % gemm::BK);
  auto kern = p.ragged ? gemm_st::gemm_st_kernel<KIND, BN, PAIR, QOUT, true>
                       : gemm_st::gemm_st_kernel<KIND, BN, PAIR, QOUT, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = ((a.M + TILE_M - 1) / TILE_M) * ((a.N + BN - 1) / BN);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(gemm_st::NUM_THREADS_ST);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0] = pdl_attribute();
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = PAIR ? 2 : 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = PAIR ? 2 : 1;
  // persistent grid: no more units than can be resident at once (pairs must
  // sit in one GPC, so fewer than SMs/2 pairs may fit)
  int units = PAIR ? sms / 2 : sms;
  if (PAIR) {
    int clusters = 0;
    cfg.gridDim = dim3((unsigned)(2 * units));
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters > 0 &&
        clusters < units)
      units = clusters;
  }
  const int grid_units = (int)(tiles < units ? tiles : units);
  cfg.gridDim = dim3((unsigned)(PAIR ? 2 * grid_units : grid_units));
  e = cudaLaunchKernelEx(&cfg, kern, ma, mb, md, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool QOUT>
static cudaError_t launch_st_any(const GemmArgs &a, cudaStream_t st) {
  // 256-wide tiles (and 256-row pairs) where they cover no more than
  // 128-wide (128-row) tiles would
  auto up = [](int64_t v, int64_t m) { return (v + m - 1) / m * m; };
  const bool wide = up(a.N, 256) == up(a.N, 128);
  const bool pair = wide && up(a.M, 256) == up(a.M, 128);
  if (a.fmt == kMX)
    return pair ? launch_st<kMX, 256, true, QOUT>(a, st)
                : (wide ? launch_st<kMX, 256, false, QOUT>(a, st) : launch_st<kMX, 128, false, QOUT>(a, st));
  return pair ? launch_st<kNVG, 256, true, QOUT>(a, st)
              : (wide ? launch_st<kNVG, 256, false, QOUT>(a, st) : launch_st<kNVG, 128, false, QOUT>(a, st));
}

cudaError_t launch_gemm_blockscaled(const GemmArgs &a, cudaStream_t st) {
  if (a.fmt == kMX || a.fmt == kNVG) {
    if (a.q_payload) {
      if (a.out_fp32) return cudaErrorInvalidValue;  // the quantized output comes from bf16 D
      return launch_st_any<true>(a, st);
    }
    if (!a.D) return cudaErrorInvalidValue;
    return launch_st_any<false>(a, st);
  }
  if (a.fmt == kNVC && !a.q_payload && a.D) {
    // 1-SM 128 x 128 tiles: measured 3-9% faster than the 2-SM 256 x 128
    // pair form on the 8B forward shapes (both are held back by the chunk
    // fold's synchronization, not by operand traffic)
    return launch_st<kNVC, 128, false, false>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace fa4
