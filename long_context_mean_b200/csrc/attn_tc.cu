// Block-sparse FlashAttention forward on the sm_100a tensor cores.
//
// [P3] SpargeAttention notes, 2.1: per query block, the kept key blocks are
// visited in ascending order with the online softmax (m, l, O); 2.3: the P V
// product of a tile is skipped when max over the block's rows of
// (rowmax S - running max) < lambda, l still counting the tile.
//
// Design (bf16, d = dv = 128, bq = 128, bk = 64 or 128):
//   * persistent grid, one CTA per SM, PIPES independent pipelines per CTA
//     (2 for bk = 64, 1 for bk = 128) so every SM sub-partition holds PIPES
//     softmax warps.  Units (b, h, q-block) are taken dynamically, in the
//     mask's work order (descending kept count), from a global counter by
//     each pipeline's producer and announced to its MMA and softmax warps
//     through a 4-slot ring.
//   * per pipeline, warp p is the TMA producer: lane 0 loads the Q tile once
//     per unit and the K tiles of the kept key blocks through a 3-stage ring,
//     lane 1 the V tiles through their own ring (a K load never waits behind
//     a V stage that the previous P V still holds).  Warp 2+p (one lane)
//     issues tcgen05.mma: S = Q K^T into one of two TMEM S buffers and
//     O += P V into the TMEM O accumulator.  The softmax writes P (bf16
//     pairs) over its S buffer in TMEM and the P V product reads it from
//     there (TS form), so S runs one tile ahead of P V: S(t+1) overlaps the
//     softmax of t, and P V(t) the softmax of t+1.  (Q copied into TMEM with
//     a TS-form S and one S buffer per pipeline measured 40% slower on B200:
//     each pipeline's chain softmax -> P V -> S becomes serial.)
//   * per pipeline, four softmax warps (one thread per query row = TMEM
//     lane): S from TMEM, masks, running max, exp2 (scale folded into one
//     packed fp32x2 FMA), P, O rescale in TMEM when the reference maximum
//     moves, the epilogue O / l and LSE (stored through an optional row
//     permutation).  Each warp publishes the largest (tile max - running
//     max) of its rows; the MMA warp combines the four and takes the lambda
//     decision, so the softmax warps never wait for one another.
//   The exact running max drives the lambda test; O and l use a reference
//   maximum that only moves when the running max exceeds it by more than
//   2^8 (O / l is the same quotient).  A row whose maximum moves has a gap of
//   0, so a tile that needs a rescale is never skipped.
// 8-bit QK ([P3] 2.4, QM = 1: INT8, 2: FP8 E4M3): Q and K tiles hold one
// code per element (one 128-byte swizzle row per token), S is four
// kind::i8 / kind::f8f6f4 steps, and the softmax multiplies each tile by its
// own scale (the two block scales of the quantisation); INT8 scores are
// int32 and reach the float path through an exact biased-float add.
// Every mbarrier wait is bounded (2 s; 10 ms under SA_FLAG_TEST_STALL); on
// expiry the kernel raises SA_ERR_TIMEOUT and sets the CTA's abort flag, after
// which every wait returns at once and every role stops issuing: the loaders
// drain the copies they issued, the MMA warp waits (bounded) for the tensor
// operations it issued, the softmax warps leave together, and the TMEM
// allocation is released.
#include <cuda.h>

#include "sa_internal.cuh"

namespace sa {
namespace {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;       // 2 s
constexpr unsigned long long kTestWaitLimitNs = 10000000ull;     // 10 ms (SA_FLAG_TEST_STALL)
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int BK, int QM>
struct Cfg {
  static constexpr int PIPES = BK == 64 ? 2 : 1;
  static constexpr int S_BUFS = 2;                    // TMEM S buffers per pipeline
  static constexpr int LOOKAHEAD = 1;                 // S tiles issued ahead of P V
  // K and V rings.  K is needed one softmax ahead of V, so it gets the deeper
  // ring: three stages everywhere (the TMA latency, about 1 us, is longer
  // than a tile); V two stages for bf16 at bk = 64 (shared memory: 2 x 112 KB)
  // and three where the tiles are smaller (8-bit Q and K) or one pipeline.
  static constexpr int K_STAGES = 3;
  static constexpr int V_STAGES = (BK == 64 && QM == 0) ? 2 : 3;
  // Softmax warps per TMEM lane quarter.  Two (16 rows each, half of a
  // row's columns per thread, 640 threads) measured 6% slower than one at
  // bk = 64 on B200, so one warp owns each quarter.
  static constexpr int SPLIT = 1;
  static constexpr int SM_WARPS = 4 * SPLIT;          // softmax warps per pipeline
  static constexpr int THREADS = 128 + 32 * SM_WARPS * PIPES;
  static constexpr int QK_ELEM = QM ? 1 : 2;           // bytes per Q / K element
  static constexpr int Q_BYTES = 128 * 128 * QK_ELEM;
  static constexpr int K_BYTES = BK * 128 * QK_ELEM;
  static constexpr int V_BYTES = BK * 128 * 2;
  static constexpr int KV_CHUNK = BK * 128;          // one 128-byte-wide chunk: BK rows x 128 B
  static constexpr int PIPE_BYTES = Q_BYTES + K_STAGES * K_BYTES + V_STAGES * V_BYTES;
  static constexpr int OFF_CTL = PIPES * PIPE_BYTES;
  static constexpr int CTL_BYTES = 512;
  static constexpr int SMEM = OFF_CTL + PIPES * CTL_BYTES + 1024;   // + alignment slack
  // TMEM columns of a pipeline: O [0, 128), then the S buffers (BK fp32
  // columns each).
  static constexpr int S_COL = 128;
  static constexpr int TMEM_PIPE = (S_COL + S_BUFS * BK) <= 256 ? 256 : 512;
  static constexpr int TMEM_COLS = PIPES * TMEM_PIPE;
  // buffer and phase of tile gt in the S / P / PV-done rings
  static __host__ __device__ constexpr int sbuf(uint32_t gt) { return (int)(gt & 1); }
  static __host__ __device__ constexpr uint32_t sphase(uint32_t gt) { return (gt >> 1) & 1; }
  static __host__ __device__ constexpr int off_q(int p) { return p * PIPE_BYTES; }
  static __host__ __device__ constexpr int off_k(int p) { return p * PIPE_BYTES + Q_BYTES; }
  static __host__ __device__ constexpr int off_v(int p) { return p * PIPE_BYTES + Q_BYTES + K_STAGES * K_BYTES; }
};

// Per-pipeline control block (8-byte mbarriers first).
struct Ctl {
  uint64_t q_full, q_empty, o_free;
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t u_full[4], u_empty[4];          // unit announcement ring
  uint64_t mma_done;                       // the MMA warp's last tensor operations have completed
  unsigned long long wait_ns;              // limit of every wait
  uint32_t tmem_base;
  volatile uint32_t abort;
  float gapw[4][8];                        // [tile & 3][softmax warp]
  // Unit announcements: the producer resolves each unit once (work-order
  // entry, list offsets) and the other roles read it from here.  i < 0 ends
  // the work.
  struct Slot {
    int32_t i, n, lo, bh, qb, kvh;
  };
  volatile Slot ring[4];
};
static_assert(sizeof(Ctl) <= 512, "control block too large");
static_assert(Cfg<64, 0>::SMEM <= 227 * 1024 && Cfg<128, 0>::SMEM <= 227 * 1024 &&
                  Cfg<64, 1>::SMEM <= 227 * 1024 && Cfg<128, 1>::SMEM <= 227 * 1024 &&
                  Cfg<64, 2>::SMEM <= 227 * 1024 && Cfg<128, 2>::SMEM <= 227 * 1024,
              "shared memory above the 227 KB a CTA may use");
static_assert(Cfg<64, 0>::K_STAGES <= 3 && Cfg<64, 0>::V_STAGES <= 3 && Cfg<128, 1>::V_STAGES <= 3,
              "the control block holds three stages per ring");
static_assert(Cfg<64, 0>::TMEM_COLS <= 512 && Cfg<128, 0>::TMEM_COLS <= 512 && Cfg<64, 1>::TMEM_COLS <= 512,
              "TMEM holds 512 columns");

struct TcParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int64_t col_capacity;
  const int32_t* order;
  uint16_t* out;
  float* lse;
  const int32_t* out_perm;
  uint8_t* skip_log;
  int32_t* status;
  int32_t* counter;      // work counter, zero at launch
  int64_t N, nqb, nkb;
  int64_t perm_stride;   // 0: one out_perm for every head; N: one per query head
  const float* tile_scale;   // 8-bit QK: log2-domain scale of each kept tile, CSR order
  int32_t Hq, Hkv;
  int32_t num_units;
  int32_t causal;
  float scale_log2;
  float lam_log2;
  unsigned long long wait_ns;   // limit of every mbarrier wait
  int32_t stall;                // test hook: CTA 0 issues no K loads (its waits run out)
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// One try_wait: the hardware may suspend the thread for a short,
// implementation-defined time until the phase completes, so waiting warps
// take few issue slots.  (An explicit suspend-time hint of 1 ms measured
// 2.4 % slower on B200: the waiting roles woke later.)
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait.  Returns false when the CTA is aborting (a wait elsewhere
// expired) or this wait expired (then it raises the abort itself).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Ctl* g, int32_t* status) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (;;) {
    if (mbar_try(bar, parity)) return true;
    if (g->abort) return false;
    if (globaltimer() - t0 > g->wait_ns) {
      g->abort = 1;
      raise_status(status, SA_ERR_TIMEOUT);
      return false;
    }
  }
}
// Bounded wait that ignores the abort flag (draining in-flight copies).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, unsigned long long limit) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try(bar, parity)) {
    if (globaltimer() - t0 > limit) return;
  }
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// D (TMEM) = A (SMEM desc) x B (SMEM desc) [+ D]
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// D (TMEM, int32) = A (SMEM desc, s8) x B (SMEM desc, s8) [+ D]
__device__ __forceinline__ void umma_ss_i8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// D (TMEM, f32) = A (SMEM desc, e4m3) x B (SMEM desc, e4m3) [+ D]
__device__ __forceinline__ void umma_ss_f8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// D (TMEM) = A (TMEM) x B (SMEM desc) [+ D]
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// 16x32bx2 shapes: 16 TMEM lanes from the lane in taddr; thread t < 16 gets
// lane t at columns [c, c + n), thread t + 16 lane t at [c + IMM, c + IMM + n).
template <int IMM>
__device__ __forceinline__ void tmem_ld_16x32bx2_x32(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], %33;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr), "n"(IMM));
}
template <int IMM>
__device__ __forceinline__ void tmem_st_16x32bx2_x32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], %1, "
      "{%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33};" ::"r"(taddr), "n"(IMM),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
template <int IMM>
__device__ __forceinline__ void tmem_ld_16x32bx2_x16(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], %17;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr), "n"(IMM));
}
template <int IMM>
__device__ __forceinline__ void tmem_st_16x32bx2_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], %1, "
      "{%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17};" ::"r"(taddr), "n"(IMM),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}
// Two fp32 values in one 64-bit register for the packed fp32x2 pipe.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 version 1).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: bf16 x bf16 -> f32, A K-major.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
// Instruction descriptor, kind::i8: s8 x s8 -> s32 (D format 2, A and B
// format 1 = signed), both operands K-major, no saturation.
__host__ __device__ constexpr uint32_t make_idesc_s8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Instruction descriptor, kind::f8f6f4: e4m3 x e4m3 -> f32 (D format 1, A
// and B format 0 = E4M3), both operands K-major.
__host__ __device__ constexpr uint32_t make_idesc_e4m3(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// An int32 in (-2^22, 2^22) as a float biased by 1.5 * 2^23: the bit pattern
// of 12582912 + x, exact (used on the raw int32 S tile of the INT8 path).
constexpr int32_t kBiasBits = 0x4B400000;
constexpr float kBias = 12582912.0f;

struct Unit {
  int64_t bh, qb, kvh;
  int64_t lo, n;
};

__device__ __forceinline__ Unit unit_at(const TcParams& p, int i, int BK) {
  Unit u;
  const int64_t id = p.order ? p.order[i] : i;
  u.bh = id / p.nqb;
  u.qb = id % p.nqb;
  const int64_t b = u.bh / p.Hq, h = u.bh % p.Hq;
  u.kvh = b * p.Hkv + h / (p.Hq / p.Hkv);
  if (p.row_ptr) {
    u.lo = p.row_ptr[id];
    const int64_t hi = p.row_ptr[id + 1];
    // A list that reaches past col_idx (the builder raised SA_ERR_CAPACITY)
    // is not computed: n = -1 tells every role to pass the unit by.
    u.n = (hi > p.col_capacity || u.lo > hi) ? -1 : hi - u.lo;
  } else {
    u.lo = 0;
    const int64_t last_row = min64(p.N, (u.qb + 1) * 128) - 1;
    u.n = p.causal ? (last_row / BK + 1) : p.nkb;
  }
  return u;
}

__device__ __forceinline__ int64_t kblock_at(const TcParams& p, const Unit& u, int64_t t) {
  return p.row_ptr ? p.col_idx[u.lo + t] : t;
}

// Publish unit i (or the end of the work, i < 0) in a ring slot; read it back.
__device__ __forceinline__ void post_unit(Ctl* c, int slot, int i, const Unit& u) {
  volatile Ctl::Slot& s = c->ring[slot];
  s.i = i;
  s.n = (int32_t)u.n;
  s.lo = (int32_t)u.lo;
  s.bh = (int32_t)u.bh;
  s.qb = (int32_t)u.qb;
  s.kvh = (int32_t)u.kvh;
}
__device__ __forceinline__ int read_unit(Ctl* c, int slot, Unit& u) {
  const volatile Ctl::Slot& s = c->ring[slot];
  u.n = s.n;
  u.lo = s.lo;
  u.bh = s.bh;
  u.qb = s.qb;
  u.kvh = s.kvh;
  return s.i;
}

// ---------------------------------------------------------------------------
// Roles
// ---------------------------------------------------------------------------
template <int BK, int QM>
__device__ void producer(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                         const TcParams& p, Ctl* c, Ctl* g, uint32_t sb, int pipe) {
  // Lane 0 claims the units and loads Q and the K tiles; it announces each
  // unit through the ring.
  using C = Cfg<BK, QM>;
  uint32_t k_it = 0, nq = 0;
  for (uint32_t j = 0;; ++j) {
    // Take the next unit of the work order and announce it to the pipeline's
    // V loader, MMA and softmax warps through a 4-slot ring.
    const int slot = j & 3;
    if (!mbar_wait(&c->u_empty[slot], ((j >> 2) & 1) ^ 1, g, p.status)) break;
    int i = atomicAdd(p.counter, 1);
    if (i >= p.num_units) i = -1;
    Unit u{};
    if (i >= 0) u = unit_at(p, i, BK);
    post_unit(c, slot, i, u);
    mbar_arrive(&c->u_full[slot]);
    if (i < 0) break;
    if (u.n <= 0) continue;
    if (!mbar_wait(&c->q_empty, (nq & 1) ^ 1, g, p.status)) break;
    ++nq;
    mbar_expect_tx(&c->q_full, C::Q_BYTES);
    tma_load_3d(sb + C::off_q(pipe), tmQ, 0, (int)(u.qb * 128), (int)u.bh, &c->q_full);
    if constexpr (QM == 0)   // bf16 rows are two 128-byte chunks; 8-bit rows one
      tma_load_3d(sb + C::off_q(pipe) + C::Q_BYTES / 2, tmQ, 64, (int)(u.qb * 128), (int)u.bh, &c->q_full);
    if (p.stall && blockIdx.x == 0) continue;   // test hook: no K tile arrives here
    bool ok = true;
    for (int64_t t = 0; t < u.n && ok; ++t) {
      const int kb = (int)kblock_at(p, u, t);
      const int s = k_it % C::K_STAGES;
      const uint32_t ph = (k_it / C::K_STAGES) & 1;
      const uint32_t kdst = sb + C::off_k(pipe) + s * C::K_BYTES;
      ok = mbar_wait(&c->k_empty[s], ph ^ 1, g, p.status);
      if (!ok) break;
      mbar_expect_tx(&c->k_full[s], C::K_BYTES);
      tma_load_3d(kdst, tmK, 0, kb * BK, (int)u.kvh, &c->k_full[s]);
      if constexpr (QM == 0) tma_load_3d(kdst + C::KV_CHUNK, tmK, 64, kb * BK, (int)u.kvh, &c->k_full[s]);
      ++k_it;
    }
    if (!ok) break;
  }
  // Drain: the last copies issued into every stage (and the last Q) have
  // landed before the CTA may exit.
  if (nq > 0) mbar_drain(&c->q_full, (nq - 1) & 1, g->wait_ns);
  for (uint32_t j = k_it > (uint32_t)C::K_STAGES ? k_it - C::K_STAGES : 0; j < k_it; ++j)
    mbar_drain(&c->k_full[j % C::K_STAGES], (j / C::K_STAGES) & 1, g->wait_ns);
}

// Lane 1 of the producer warp loads the V tiles on their own ring, so a K
// load never waits behind a V stage that the previous P V still holds.
template <int BK, int QM>
__device__ void v_loader(const CUtensorMap* tmV, const TcParams& p, Ctl* c, Ctl* g, uint32_t sb, int pipe) {
  using C = Cfg<BK, QM>;
  uint32_t v_it = 0;
  for (uint32_t j = 0;; ++j) {
    const int slot = j & 3;
    if (!mbar_wait(&c->u_full[slot], (j >> 2) & 1, g, p.status)) break;
    Unit u;
    const int i = read_unit(c, slot, u);
    mbar_arrive(&c->u_empty[slot]);
    if (i < 0) break;
    bool ok = true;
    for (int64_t t = 0; t < u.n; ++t) {
      const int kb = (int)kblock_at(p, u, t);
      const int s = v_it % C::V_STAGES;
      const uint32_t ph = (v_it / C::V_STAGES) & 1;
      const uint32_t vdst = sb + C::off_v(pipe) + s * C::V_BYTES;
      ok = mbar_wait(&c->v_empty[s], ph ^ 1, g, p.status);
      if (!ok) break;
      mbar_expect_tx(&c->v_full[s], C::V_BYTES);
      tma_load_3d(vdst, tmV, 0, kb * BK, (int)u.kvh, &c->v_full[s]);
      tma_load_3d(vdst + C::KV_CHUNK, tmV, 64, kb * BK, (int)u.kvh, &c->v_full[s]);
      ++v_it;
    }
    if (!ok) break;
  }
  for (uint32_t j = v_it > (uint32_t)C::V_STAGES ? v_it - C::V_STAGES : 0; j < v_it; ++j)
    mbar_drain(&c->v_full[j % C::V_STAGES], (j / C::V_STAGES) & 1, g->wait_ns);
}

template <int BK, int QM>
__device__ void mma_issuer(const TcParams& p, Ctl* c, Ctl* g, uint32_t sb, uint32_t tm, int pipe) {
  using C = Cfg<BK, QM>;
  constexpr uint32_t idesc_s =
      QM == 1 ? make_idesc_s8(128, BK) : (QM == 2 ? make_idesc_e4m3(128, BK) : make_idesc(128, BK, 0));
  constexpr uint32_t idesc_pv = make_idesc(128, 128, 1);
  uint32_t kv_it = 0, gt0 = 0, unit_it = 0;   // unit_it counts units with work
  bool ok = true;                             // false once a wait gave up: issue nothing more
  for (uint32_t j = 0; ok; ++j) {
    const int slot = j & 3;
    if (!(ok = mbar_wait(&c->u_full[slot], (j >> 2) & 1, g, p.status))) break;
    Unit u;
    const int i = read_unit(c, slot, u);
    mbar_arrive(&c->u_empty[slot]);
    if (i < 0) break;
    if (u.n <= 0) continue;
    if (!(ok = mbar_wait(&c->q_full, unit_it & 1, g, p.status))) break;
    tc_fence_after();
    const uint32_t qbase = sb + C::off_q(pipe);
    bool first_pv = true;
    auto do_pv = [&](int64_t tt) {
      if (!ok) return;
      const uint32_t it = kv_it + (uint32_t)tt, gt = gt0 + (uint32_t)tt;
      const int s = it % C::V_STAGES;
      const uint32_t ph = (it / C::V_STAGES) & 1;
      const int gb = C::sbuf(gt);
      if (!(ok = mbar_wait(&c->p_full[gb], C::sphase(gt), g, p.status))) return;
      tc_fence_after();
      const float* gw = c->gapw[gt & 3];
      float gmax = gw[0];
#pragma unroll
      for (int w = 1; w < C::SM_WARPS; ++w) gmax = fmaxf(gmax, gw[w]);
      const bool skip = gmax < p.lam_log2;
      if (p.skip_log && p.row_ptr) p.skip_log[u.lo + tt] = skip ? 1 : 0;
      if (tt == 0) {
        if (!(ok = mbar_wait(&c->o_free, (unit_it & 1) ^ 1, g, p.status))) return;
        tc_fence_after();
      }
      if (!(ok = mbar_wait(&c->v_full[s], ph, g, p.status))) return;
      tc_fence_after();
      if (!skip) {
        const uint32_t vbase = sb + C::off_v(pipe) + s * C::V_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t b = desc_sw128(vbase + kk * 2048, C::KV_CHUNK, 1024);
          const uint32_t acc = (first_pv && kk == 0) ? 0u : 1u;
          umma_ts(tm, tm + C::S_COL + gb * BK + kk * 8, b, idesc_pv, acc);   // P over the S buffer
        }
        first_pv = false;
      }
      umma_commit(&c->v_empty[s]);
      umma_commit(&c->pv_done[gb]);
    };
    for (int64_t t = 0; t < u.n && ok; ++t) {
      const uint32_t it = kv_it + (uint32_t)t, gt = gt0 + (uint32_t)t;
      const int s = it % C::K_STAGES;
      const uint32_t ph = (it / C::K_STAGES) & 1;
      const uint32_t scol = tm + C::S_COL + C::sbuf(gt) * BK;
      if (!(ok = mbar_wait(&c->k_full[s], ph, g, p.status))) break;
      tc_fence_after();
      const uint32_t kbase = sb + C::off_k(pipe) + s * C::K_BYTES;
      if constexpr (QM != 0) {
        // d = 128 8-bit codes = one 128-byte swizzle row; K = 32 per instruction.
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t a = desc_sw128(qbase + kk * 32, 16, 1024);
          const uint64_t b = desc_sw128(kbase + kk * 32, 16, 1024);
          if constexpr (QM == 1)
            umma_ss_i8(scol, a, b, idesc_s, kk > 0 ? 1u : 0u);
          else
            umma_ss_f8(scol, a, b, idesc_s, kk > 0 ? 1u : 0u);
        }
      } else {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = desc_sw128(qbase + (kk >> 2) * (C::Q_BYTES / 2) + (kk & 3) * 32, 16, 1024);
          const uint64_t b = desc_sw128(kbase + (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32, 16, 1024);
          umma_ss(scol, a, b, idesc_s, kk > 0 ? 1u : 0u);
        }
      }
      umma_commit(&c->s_full[C::sbuf(gt)]);
      umma_commit(&c->k_empty[s]);
      if (t == u.n - 1) umma_commit(&c->q_empty);
      if (t >= C::LOOKAHEAD) do_pv(t - C::LOOKAHEAD);
    }
    for (int64_t tt = u.n > C::LOOKAHEAD ? u.n - C::LOOKAHEAD : 0; tt < u.n; ++tt) do_pv(tt);
    kv_it += (uint32_t)u.n;
    gt0 += (uint32_t)u.n;
    ++unit_it;
  }
  // Every tensor operation this thread issued has completed before the TMEM
  // allocation can be released (on the normal path they already have).
  umma_commit(&c->mma_done);
  mbar_drain(&c->mma_done, 0, g->wait_ns);
}

// Largest value of a float over the warp (order-preserving int key).
__device__ __forceinline__ float warp_fmax(float v) {
  int k = __float_as_int(v);
  k = k >= 0 ? k : k ^ 0x7FFFFFFF;
  const int m = __reduce_max_sync(0xffffffffu, k);
  return __int_as_float(m >= 0 ? m : m ^ 0x7FFFFFFF);
}

// One softmax thread holds NC = BK / SPLIT score columns of one query row.
// SPLIT = 1: a warp owns the 32 rows (TMEM lanes) of its quarter, one row a
// thread (32x32b shapes).  SPLIT = 2: two warps share a quarter, 16 rows
// each; threads t and t + 16 hold columns [0, NC) and [NC, 2 NC) of the same
// row (16x32bx2 shapes), so the row's maximum and sum take one shuffle.
template <int BK, int QM>
__device__ void softmax_rows(const TcParams& p, Ctl* c, Ctl* g, uint32_t tm, int wq, int half, int lane) {
  using C = Cfg<BK, QM>;
  constexpr int SPLIT = C::SPLIT;
  constexpr int NC = BK / SPLIT;                                  // score columns per thread
  const int rlane = SPLIT == 2 ? half * 16 + (lane & 15) : lane;  // TMEM lane within the quarter
  const int row = wq * 32 + rlane;
  const int cpart = SPLIT == 2 ? (lane >> 4) : 0;                 // which column part of the row
  const uint32_t lane_off = (uint32_t)(wq * 32 + (SPLIT == 2 ? half * 16 : 0)) << 16;
  const int widx = wq * SPLIT + half;                              // this warp among the pipeline's
  const bool row_owner = SPLIT == 1 || lane < 16;                  // one thread per row stores LSE
  float sc = p.scale_log2;   // log2-domain score scale; 8-bit QK: per tile
  uint32_t gt0 = 0;
  for (uint32_t j = 0;; ++j) {
    const int slot = j & 3;
    // A wait that gives up (the CTA is aborting) ends the warp's work; the
    // decision is warp-uniform, as tcgen05.ld/st are warp-collective.
    if (!__all_sync(0xffffffffu, mbar_wait(&c->u_full[slot], (j >> 2) & 1, g, p.status))) return;
    Unit u;
    const int i = read_unit(c, slot, u);
    __syncwarp();
    if (lane == 0) mbar_arrive(&c->u_empty[slot]);
    if (i < 0) break;
    const int64_t row_g = u.qb * 128 + row;
    const bool row_valid = row_g < p.N;
    // The row's destination (the inverse reorder), fetched now so that the
    // load is long done when the epilogue stores through it.
    const int64_t out_row =
        row_valid ? (p.out_perm ? (int64_t)p.out_perm[u.bh * p.perm_stride + row_g] : row_g) : 0;
    if (u.n <= 0) {
      if (row_valid && row_owner) raise_status(p.status, u.n < 0 ? SA_ERR_CAPACITY : SA_ERR_EMPTY_ROW);
      continue;
    }
    // m_run, m_ref are the row's (equal in both threads of a row); l is this
    // thread's part of the row sum.
    float m_run = -INFINITY, m_ref = -INFINITY, l = 0.f;
    int64_t kb_cur = kblock_at(p, u, 0);
    float sc_next = 0.f;
    if constexpr (QM != 0) sc_next = p.tile_scale[u.lo];
    for (int64_t t = 0; t < u.n; ++t) {
      const uint32_t gt = gt0 + (uint32_t)t;
      const int gb = C::sbuf(gt);
      const uint32_t scol = tm + lane_off + C::S_COL + gb * BK;
      const int64_t kb_next = (t + 1 < u.n) ? kblock_at(p, u, t + 1) : 0;   // load ahead
      if constexpr (QM != 0) {
        sc = sc_next;
        if (t + 1 < u.n) sc_next = p.tile_scale[u.lo + t + 1];
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&c->s_full[gb], C::sphase(gt), g, p.status))) return;
      tc_fence_after();
      float s[NC];
      if constexpr (SPLIT == 2) {
        tmem_ld_16x32bx2_x32<NC>(scol, s);
      } else {
#pragma unroll
        for (int cc = 0; cc < NC / 32; ++cc) tmem_ld32(scol + cc * 32, s + cc * 32);
      }
      tmem_wait_ld();
      if constexpr (QM == 1) {
        // int32 scores -> floats biased by kBias (exact); the bias cancels
        // in the exponent offset and the tile maximum below.
#pragma unroll
        for (int jj = 0; jj < NC; ++jj) s[jj] = __int_as_float(__float_as_int(s[jj]) + kBiasBits);
      }

      const int64_t kt0 = kb_cur * BK;            // first key of the tile
      kb_cur = kb_next;
      const int64_t k0 = kt0 + cpart * NC;        // key of this thread's first column
      const bool need_mask = (kt0 + BK > p.N) || (p.causal && kt0 + BK - 1 > u.qb * 128);
      if (need_mask) {
#pragma unroll
        for (int jj = 0; jj < NC; ++jj) {
          const int64_t key = k0 + jj;
          if (key >= p.N || (p.causal && key > row_g)) s[jj] = -INFINITY;
        }
      }
      // P = exp2(s * scale_log2 - ref), packed to bf16 pairs, and its sum.
      uint32_t pk[NC / 2];
      float row_sum = 0.f;
      auto compute_p = [&](float ref) {
        // Pairs of columns on the packed fp32x2 pipe: x = s * scale - ref.
        const float off = QM == 1 ? fmaf(-kBias, sc, -ref) : -ref;
        const uint64_t sc2 = pack2(sc, sc), neg2 = pack2(off, off);
        uint64_t acc[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[jj] = pack2(0.f, 0.f);
#pragma unroll
        for (int jj = 0; jj < NC; jj += 2) {
          const uint64_t x = ffma2(pack2(s[jj], s[jj + 1]), sc2, neg2);
          float x0, x1;
          unpack2(x, x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          acc[(jj >> 1) & 3] = fadd2(acc[(jj >> 1) & 3], pack2(p0, p1));
          pk[jj >> 1] = pack_bf16(p0, p1);
        }
        const uint64_t a2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
        float lo, hi;
        unpack2(a2, lo, hi);
        row_sum = lo + hi;
      };
      // Speculate with the current reference maximum: P needs the tile's
      // maximum only when that maximum exceeds the reference by more than
      // the threshold (then P is recomputed below), so the exponentials and
      // the max tree are independent work.
      const bool spec = m_ref > -INFINITY;
      if (spec) compute_p(m_ref);
      // Row max as a tree of 3-input maxima (independent chains), raw units.
      float mx[NC / 4];
#pragma unroll
      for (int jj = 0; jj < NC / 4; ++jj) mx[jj] = max3(fmaxf(s[4 * jj], s[4 * jj + 1]), s[4 * jj + 2], s[4 * jj + 3]);
#pragma unroll
      for (int w = NC / 4; w > 1; w = (w + 2) / 3) {
#pragma unroll
        for (int jj = 0; jj < (w + 2) / 3; ++jj) {
          const float a = mx[3 * jj];
          const float b = 3 * jj + 1 < w ? mx[3 * jj + 1] : a;
          const float d = 3 * jj + 2 < w ? mx[3 * jj + 2] : a;
          mx[jj] = max3(a, b, d);
        }
      }
      float mraw = mx[0];
      if constexpr (SPLIT == 2) mraw = fmaxf(mraw, __shfl_xor_sync(0xffffffffu, mraw, 16));
      const float mloc = (QM == 1 ? mraw - kBias : mraw) * sc;   // scale > 0: max commutes
      const float m_new = fmaxf(m_run, mloc);
      const float gap = warp_fmax((row_valid && mloc > -INFINITY) ? mloc - m_new : -INFINITY);
      if (lane == 0) c->gapw[gt & 3][widx] = gap;
      m_run = m_new;
      float corr = 1.f;
      bool resc = false;
      if (m_new > -INFINITY && (m_ref == -INFINITY || m_new > m_ref + kRescaleThreshold)) {
        corr = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);
        m_ref = m_new;
        resc = (t > 0);
        compute_p(m_ref);                       // the speculation missed
      } else if (!spec) {
#pragma unroll
        for (int jj = 0; jj < NC / 2; ++jj) pk[jj] = 0u;   // every score so far masked
        row_sum = 0.f;
      }
      l = l * corr + row_sum;
      // tcgen05.ld/st are warp-collective: a warp rescales when any of its
      // rows needs it (corr is 1 for the others).  A rescale implies the
      // tile is not skipped, so PV(t-1) is the last product to wait for.
      if (__any_sync(0xffffffffu, resc)) {
        const uint32_t gp = gt - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&c->pv_done[C::sbuf(gp)], C::sphase(gp), g, p.status))) return;
        tc_fence_after();
        const float f = resc ? corr : 1.f;
        if constexpr (SPLIT == 2) {
          // this thread's 64 columns of the row, 16 at a time
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            float o[16];
            tmem_ld_16x32bx2_x16<64>(tm + lane_off + cc * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) o[jj] *= f;
            tmem_st_16x32bx2_x16<64>(tm + lane_off + cc * 16, reinterpret_cast<const uint32_t*>(o));
          }
        } else {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float o[32];
            tmem_ld32(tm + lane_off + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) o[jj] *= f;
            tmem_st32(tm + lane_off + cc * 32, reinterpret_cast<const uint32_t*>(o));
          }
        }
        tmem_wait_st();
      }
      if constexpr (SPLIT == 2) {
        tmem_st_16x32bx2_x16<NC / 2>(scol, pk);   // P over the first BK / 2 columns of S
      } else {
#pragma unroll
        for (int cc = 0; cc < BK / 64; ++cc) tmem_st32(scol + cc * 32, pk + cc * 32);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&c->p_full[gb]);
    }
    // Epilogue: O / l from TMEM once the unit's last PV has landed.
    const uint32_t gl = gt0 + (uint32_t)u.n - 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&c->pv_done[C::sbuf(gl)], C::sphase(gl), g, p.status))) return;
    tc_fence_after();
    if constexpr (SPLIT == 2) l += __shfl_xor_sync(0xffffffffu, l, 16);   // the row's two parts
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    // SPLIT = 2: this thread stores the row's output columns [64 cpart, 64 cpart + 64).
    uint16_t* orow = p.out + (u.bh * p.N + out_row) * 128 + cpart * 64;
    constexpr int OCH = SPLIT == 2 ? 16 : 32;   // output columns per TMEM load
#pragma unroll
    for (int cc = 0; cc < 128 / SPLIT / OCH; ++cc) {
      float o[OCH];
      if constexpr (SPLIT == 2)
        tmem_ld_16x32bx2_x16<64>(tm + lane_off + cc * OCH, o);
      else
        tmem_ld32(tm + lane_off + cc * OCH, o);
      tmem_wait_ld();
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow + cc * OCH);
#pragma unroll
        for (int q4 = 0; q4 < OCH / 8; ++q4) {
          uint4 v;
          v.x = pack_bf16(o[8 * q4 + 0] * inv_l, o[8 * q4 + 1] * inv_l);
          v.y = pack_bf16(o[8 * q4 + 2] * inv_l, o[8 * q4 + 3] * inv_l);
          v.z = pack_bf16(o[8 * q4 + 4] * inv_l, o[8 * q4 + 5] * inv_l);
          v.w = pack_bf16(o[8 * q4 + 6] * inv_l, o[8 * q4 + 7] * inv_l);
          dst[q4] = v;
        }
      }
    }
    tc_fence_before();
    mbar_arrive(&c->o_free);
    if (row_valid && row_owner) {
      if (!(l > 0.f)) raise_status(p.status, SA_ERR_EMPTY_ROW);
      if (p.lse) p.lse[u.bh * p.N + out_row] = (m_ref + __log2f(l)) * kLn2;
    }
    gt0 += (uint32_t)u.n;
  }
}

template <int BK, int QM>
__global__ void __launch_bounds__(Cfg<BK, QM>::THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, TcParams p) {
  using C = Cfg<BK, QM>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  Ctl* ctl0 = reinterpret_cast<Ctl*>(smem + C::OFF_CTL);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int q = 0; q < C::PIPES; ++q) {
      Ctl* c = reinterpret_cast<Ctl*>(smem + C::OFF_CTL + q * C::CTL_BYTES);
      mbar_init(&c->q_full, 1);
      mbar_init(&c->q_empty, 1);
      mbar_init(&c->o_free, 32 * C::SM_WARPS);
      for (int s = 0; s < C::K_STAGES; ++s) {
        mbar_init(&c->k_full[s], 1);
        mbar_init(&c->k_empty[s], 1);
      }
      for (int s = 0; s < C::V_STAGES; ++s) {
        mbar_init(&c->v_full[s], 1);
        mbar_init(&c->v_empty[s], 1);
      }
      for (int b = 0; b < C::S_BUFS; ++b) {
        mbar_init(&c->s_full[b], 1);
        mbar_init(&c->p_full[b], 32 * C::SM_WARPS);
        mbar_init(&c->pv_done[b], 1);
      }
      for (int r = 0; r < 4; ++r) {
        mbar_init(&c->u_full[r], 1);
        mbar_init(&c->u_empty[r], 2 + C::SM_WARPS);   // the V lane, the MMA lane, one lane per softmax warp
      }
      mbar_init(&c->mma_done, 1);
      c->wait_ns = p.wait_ns;
      c->abort = 0;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&ctl0->tmem_base)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl0->tmem_base;

  if (warp < 2) {
    if (warp < C::PIPES && lane < 2) {
      Ctl* c = reinterpret_cast<Ctl*>(smem + C::OFF_CTL + warp * C::CTL_BYTES);
      if (lane == 0)
        producer<BK, QM>(&tmQ, &tmK, &tmV, p, c, ctl0, sb, warp);
      else
        v_loader<BK, QM>(&tmV, p, c, ctl0, sb, warp);
    }
  } else if (warp < 4) {
    const int pipe = warp - 2;
    if (pipe < C::PIPES && lane == 0) {
      Ctl* c = reinterpret_cast<Ctl*>(smem + C::OFF_CTL + pipe * C::CTL_BYTES);
      mma_issuer<BK, QM>(p, c, ctl0, sb, tmem + pipe * C::TMEM_PIPE, pipe);
    }
    __syncwarp();
  } else {
    // Softmax warp 4 + 4 (SPLIT pipe + half) + quarter: the quarter is warp % 4,
    // the TMEM lanes a warp may access.
    const int sw = warp - 4;
    const int pipe = sw / C::SM_WARPS;
    const int half = (sw >> 2) % C::SPLIT;
    Ctl* c = reinterpret_cast<Ctl*>(smem + C::OFF_CTL + pipe * C::CTL_BYTES);
    softmax_rows<BK, QM>(p, c, ctl0, tmem + pipe * C::TMEM_PIPE, warp & 3, half, lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 3-D map over [heads][N][128] elements of 2 (bf16) or 1 (8-bit codes) bytes, box
// [1][rows][one 128-byte chunk], 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t heads, int64_t N, int rows, int elem = 2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)N, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)128 * elem, (cuuint64_t)N * 128 * elem};
  cuuint32_t box[3] = {(cuuint32_t)(128 / elem), (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BK, int QM>
sa_status launch_bk(const AttnArgs& a, cudaStream_t st) {
  using C = Cfg<BK, QM>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, a.B * a.Hq, a.N, 128, C::QK_ELEM) || !make_map(&mk, a.k, a.B * a.Hkv, a.N, BK, C::QK_ELEM) ||
      !make_map(&mv, a.v, a.B * a.Hkv, a.N, BK))
    return set_error(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point unavailable or bad map)");
  TcParams p;
  p.row_ptr = a.row_ptr;
  p.col_idx = a.col_idx;
  p.col_capacity = a.col_capacity;
  p.order = a.order;
  p.out = static_cast<uint16_t*>(a.out);
  p.lse = a.lse;
  p.out_perm = a.out_perm;
  p.perm_stride = a.perm_stride;
  p.tile_scale = a.tile_scale;
  p.skip_log = a.skip_log;
  p.status = a.status;
  p.counter = a.counter;
  p.N = a.N;
  p.nqb = a.nqb;
  p.nkb = a.nkb;
  p.Hq = (int32_t)a.Hq;
  p.Hkv = (int32_t)a.Hkv;
  p.num_units = (int32_t)(a.B * a.Hq * a.nqb);
  p.causal = a.causal;
  p.scale_log2 = a.scale * kLog2e;
  p.lam_log2 = a.lambda * kLog2e;
  p.stall = (a.flags & SA_FLAG_TEST_STALL) ? 1 : 0;
  p.wait_ns = p.stall ? kTestWaitLimitNs : kWaitLimitNs;
  if (p.num_units == 0) return SA_OK;
  if (cudaMemsetAsync(p.counter, 0, sizeof(int32_t), st) != cudaSuccess)
    return set_error(SA_ERR_CUDA, "cudaMemsetAsync(work counter) failed");
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaFuncSetAttribute(attn_tc_kernel<BK, QM>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
      cudaSuccess)
    return set_error(SA_ERR_CUDA, "cudaFuncSetAttribute(attn_tc_kernel) failed");
  const int want = (p.num_units + C::PIPES - 1) / C::PIPES;
  const int grid = want < sms ? want : sms;
  attn_tc_kernel<BK, QM><<<grid, C::THREADS, C::SMEM, st>>>(mq, mk, mv, p);
  return check_launch("attn_tc_kernel");
}

}  // namespace

bool attn_tc_supported(const sa_shape& s, int bq, int bk) {
  return s.dtype == SA_BF16 && s.d == 128 && s.dv == 128 && bq == 128 && (bk == 64 || bk == 128);
}

sa_status launch_attn_tc(const AttnArgs& a, cudaStream_t st) {
  if ((uintptr_t)a.q % 16 || (uintptr_t)a.k % 16 || (uintptr_t)a.v % 16 || (uintptr_t)a.out % 16)
    return set_error(SA_ERR_INVALID_ARG, "tensor-core path needs 16-byte aligned q, k, v, out");
  if (a.tile_scale && a.qfmt == SA_Q_E4M3) return a.bk == 64 ? launch_bk<64, 2>(a, st) : launch_bk<128, 2>(a, st);
  if (a.tile_scale) return a.bk == 64 ? launch_bk<64, 1>(a, st) : launch_bk<128, 1>(a, st);
  return a.bk == 64 ? launch_bk<64, 0>(a, st) : launch_bk<128, 0>(a, st);
}

}  // namespace sa
