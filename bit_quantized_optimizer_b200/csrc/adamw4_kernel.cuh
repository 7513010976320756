// adamw4_kernel.cuh -- the device side of the fused 4-bit AdamW step (ZIP-SR /
// ZE-EDEN) for B200 (sm_100a): constants, the structures the host fills in,
// PTX wrappers, the per-value arithmetic and the step kernel.  Included once,
// by adamw4.cu, which holds the C ABI.
//
// One kernel launch covers a range of units of a flat unit list: each block
// of a 4-bit tensor is one unit, and each fp32-state tensor is cut into
// 128-element chunks.  The grid is persistent (SM count x resident CTAs) and
// tiles of 16 consecutive units are dealt out round-robin, so all SMs stream
// one contiguous window of HBM.
//
// A CTA has one producer warp and four consumer warps, and a ring of kStages
// CTA-wide stages, one tile each.  Eight lanes take one unit, sixteen values
// per lane (two groups of eight, 64 values apart), so a warp takes four units
// and the CTA's 16 slots one tile.  For every unit of a tile, producer lane i
// writes a 64-byte header (addresses, block index, tensor id, flags, decay)
// into the stage; for runs of whole 4-bit blocks of one tensor the first lane
// of the run fills the stage with TMA bulk copies (cp.async.bulk: the run's
// fp32 or bf16 weights, bf16 grads and codes) and every lane copies its two
// block scales with 4-byte cp.async, all completing on the stage's "full"
// mbarrier.  The consumer lanes of slot i wait on it, compute unit i from the
// stage, store the results straight to global memory and hand the stage back
// on its "empty" mbarrier.  Units that are not whole 4-bit blocks (a ragged
// last block, fp32-state chunks) carry only the header and are read from
// global memory by their lanes.  Every wait is bounded by a timer; on expiry
// the kernel records the failure in a status word and the waiting warp
// leaves (the producer after draining its copies).
//
// Per unit, following the method flowchart of "ZIP-SR / ZE-EDEN: 4-bit AdamW
// state quantization" (daiwk.github.io, Method): decode the prior moments,
// update them, update the weights, requantise (ZIP-SR, ZE-EDEN or a
// state-space variant for v, NF4 for m), pack.  The weights use the
// unquantised working moments (same page, Core equation: weights are updated
// before the moments are quantised).
//
// Arithmetic follows one fixed binary32 evaluation order with IEEE division
// and square root (__fdiv_rn, __fsqrt_rn) and fused multiply-add only where
// written (__fmaf_rn, or __ffma2_rn on value pairs, which rounds each lane like
// __fmaf_rn); the library is built with -fmad=false so nothing else is
// contracted.  With that, codes, scales and weights are reproducible bit for
// bit by any IEEE implementation of the same order.
//
// No tensor cores: the step is a streaming codec (HBM is its roofline; this
// implementation is bound by instruction issue).  No TMA multicast: every
// copy is this GPU's global memory into its own CTA.
#pragma once

#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "../../include/adamw4.h"
#include "exact_math.cuh"

namespace {

constexpr int kBlock = ADAMW4_BLOCK;              // values per quantisation block
// A lane holds kSub groups of kGroup consecutive values of one block, the
// groups kBlock / kSub values apart: lane l of a block's kLanesPerUnit lanes
// takes values [64 s + 8 l, 64 s + 8 l + 8) for s = 0, 1.  A group is one
// 32-bit code word and two Philox calls.
constexpr int kGroup = 8;
constexpr int kSub = 2;
constexpr int kLanesPerUnit = kBlock / (kGroup * kSub);   // 8 lanes per block
constexpr int kUnitsPerWarp = 32 / kLanesPerUnit;         // 4 blocks per warp
constexpr int kConsumerWarps = 4;
constexpr int kConsumerThreads = 32 * kConsumerWarps;
constexpr int kCtaThreads = kConsumerThreads + 32;  // plus the producer warp
constexpr int kTileUnits = kConsumerThreads / kLanesPerUnit;  // units per tile: 16
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kStages = 3;                        // tiles in flight per CTA
// Three CTAs of five warps per SM: at most four warps per SM sub-partition,
// whose 16,384-register file then gives each thread up to 128 registers.
constexpr int kMinCtasPerSm = 3;
static_assert(kGroup * kSub * kLanesPerUnit == kBlock, "lane layout");
static_assert(kTileUnits <= 32, "one producer lane per unit");
// Value offset of group s of lane l within its block.
__host__ __device__ constexpr int group_off(int s, int l) { return s * (kBlock / kSub) + l * kGroup; }
// A tile is kTileUnits consecutive units; stage layout (CTA-wide):
//   unit headers (64 B each) | w 512 B each | g 256 B each |
//   m codes 64 B each | v codes 64 B each | m scales 8 B each | v scales 8 B each
// (each scale twice, as the pair the f32x2 decode multiplies by)
constexpr int kOffHdr = 0;
constexpr int kOffW = kOffHdr + kTileUnits * 64;
constexpr int kOffG = kOffW + kTileUnits * 512;
constexpr int kOffMC = kOffG + kTileUnits * 256;
constexpr int kOffVC = kOffMC + kTileUnits * 64;
constexpr int kOffMS = kOffVC + kTileUnits * 64;
constexpr int kOffVS = kOffMS + kTileUnits * 8;
constexpr int kStageBytes = kOffVS + kTileUnits * 8; // 15,616 B, a 16-byte multiple
constexpr uint32_t kUnitTx = 896;                 // bulk-copied bytes of one whole block
constexpr int kSmemStages = kStages * kStageBytes;
static_assert(kStageBytes % 16 == 0, "stage alignment");
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait
constexpr uint64_t kDrainLimitNs = 100000000ull;  // 0.1 s per stage when leaving early
constexpr int kVZip = ADAMW4_V_ZIPSR;
constexpr int kVZe = ADAMW4_V_ZEEDEN;
constexpr int kVZiRtn = ADAMW4_V_ZI_RTN;
constexpr int kVZiSr = ADAMW4_V_ZI_SR;
constexpr int kVZeFloor = ADAMW4_V_ZE_FLOOR;
constexpr int kVZip32 = ADAMW4_V_ZIPSR_U32;
constexpr uint32_t kBf16W = ADAMW4_T_BF16_PARAM;  // weights stored as bf16
constexpr uint32_t kKindFp32 = 1u << 16;          // internal flag: fp32-state tensor
constexpr uint32_t kStaged = 1u << 17;            // internal flag: unit data is in the stage
constexpr uint32_t kNoUnit = 1u << 18;            // internal flag: empty slot of the last tile
constexpr uint32_t kStreamV = 0u;                 // Philox stream of the v draw
constexpr uint32_t kStreamM = 1u;                 // Philox stream of the LM-head m draw
constexpr float kMagic = 12582912.0f;             // 1.5 * 2^23: adding it rounds to an integer

// Philox4x32-10 round multipliers (Salmon et al., SC'11).  The per-round keys
// (key + r * Weyl constants) are formed on the host.
constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

// One parameter tensor as the kernel sees it (64 bytes).
struct __align__(16) DevTensor {
  float* param;
  const uint16_t* grad;
  int64_t numel;
  int64_t unit_begin;   // first unit of this tensor in the flat unit list
  int64_t unit_end;     // one past its last unit
  int64_t state_off;    // 4-bit: first block in the code arena; fp32: first element
  uint32_t tensor_id;
  uint32_t flags;       // ADAMW4_T_* | kKindFp32
  float weight_decay;
  uint32_t block_offset;  // elem_offset / 128: where this piece starts in its tensor
};
static_assert(sizeof(DevTensor) == 64, "DevTensor layout");

// Per-step scalars, formed on the host in binary64 and rounded once.
struct StepArgs {
  float step_size;   // lr / (1 - b1^t)
  float rs_bc2;      // 1 / sqrt(1 - b2^t)
  float b1, omb1, b2, omb2, eps, lr;
  float nstep;                  // -step_size
  // Operand ranges of the fast division and square root (exact_math.cuh):
  // a lane takes them when all its |m1| lie in [m_lo, m_hi] and all its v1
  // in [v_lo, v_hi]; otherwise it uses the IEEE operations.  m_hi < 0
  // switches the fast path off (eps or rs_bc2 outside the range it needs).
  float m_lo, m_hi, v_lo, v_hi;
  // The broadcast operands of the f32x2 instructions, duplicated into pairs
  // here so that the instructions read them from the kernel parameters
  // instead of rebuilding a register pair for each use.
  float2 p_b1, p_omb1, p_nb2, p_nomb2, p_rs, p_eps, p_neps, p_nstep;
  float2 k_half, k_one, k_zero, k_m1, k_15, k_16, k_4096, k_magic, k_magic4096,
      k_nmagic_16, k_1_16, k_2m32, k_ze_scale0, k_ze_off0, k_ze_scale1, k_ze_off1;
  uint32_t rk0[10], rk1[10];  // Philox round keys of the seed
  uint32_t r0_hi_k0, r0_lo;   // round 0 with counter word 2 = t: hi(M1 t) ^ key0, lo(M1 t)
  int lm_sr_active;      // final-10% LM-head phase
  uint32_t* status;      // device status word (bit 0: a pipeline wait timed out;
                         // bit 1: checked build, unit out of range; bit 2: a
                         // non-finite updated weight)
  int fault_stall;       // test hook: mark stages filled without filling them
};

// The code tables' source values, formed on the host (the shared-memory
// tables SmemTables below are built from them).
struct CodeTables {
  float nf4[16];        // NF4 levels, ascending
  float nf4_gap[16];    // nf4[j+1] - nf4[j]
  float vz[16];         // ZIP-SR code points k/15
  float vz_sqrt[16];    // sqrt(k/15)
  float vz_mid[16];     // nearest-point thresholds of the k/15 code (15 used)
  float2 rtn[128];      // NF4 nearest-level buckets (floor(round(4096x + 4096)/128)):
                        // .x threshold, .y base code (int bits)
};

struct StateArena {
  uint8_t* mcodes;   // 64 bytes per block, element 2i in the low nibble of byte i
  uint8_t* vcodes;
  float* mscale;     // one per block
  float* vscale;
  float* fm;         // fp32-state tensors
  float* fv;
  int64_t nblocks4;  // blocks in the code and scale arrays (checked builds test against it)
  int64_t n32;       // elements in fm and fv (likewise)
  int64_t vs_minus_ms;  // vscale - mscale, in floats
};

// What the producer tells the consumer about one unit (64 bytes).
// The addresses are formed by the producer (one lane per unit) so that the
// consumers' eight lanes do not each recompute them.
struct __align__(16) UnitHeader {
  float* w;              // the unit's first weight (fp32, or bf16 bit patterns)
  uint32_t* mc;          // 4-bit: the block's m code words; fp32 state: its first m
  uint32_t* vc;          // 4-bit: the block's v code words; fp32 state: its first v
  float* ms;             // 4-bit: the block's m scale (its v scale: ms + vs_minus_ms)
  uint64_t e0;           // index of the unit's first element within its (logical) tensor
  uint32_t tensor_id;
  uint32_t flags;        // ADAMW4_T_* | kKindFp32 | kStaged
  float decay;           // 1 - lr * weight_decay of the tensor
  uint32_t nv_soff;      // values in the unit (bits 0-7: 1..128) | bf16-weight units:
                         // stage offset of the unit's weights << 8
  const uint16_t* g;     // its first gradient (read from global memory by direct units)
};
static_assert(sizeof(UnitHeader) == 64, "UnitHeader layout");

// ---------------------------------------------------------------------------
// PTX wrappers: mbarrier, bulk copies, timer
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for a barrier phase; false if `limit_ns` passed first.  The timer is
// read once per 64 polls.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// mbarrier.try_wait with a suspend-time hint: the thread sleeps in hardware
// until the phase completes or about `ns` nanoseconds pass, issuing nothing
// meanwhile.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// The producer's wait for a stage to come back: the consumers take
// microseconds per tile, so it sleeps in the barrier wait (20 us per try)
// instead of polling, which would take issue slots from the consumer warps
// of its SM sub-partition.  False if `limit_ns` passed first.
__device__ __forceinline__ bool wait_phase_suspended(uint32_t bar, uint32_t parity,
                                                   uint64_t limit_ns) {
  if (mbar_try_wait_suspend(bar, parity, 20000u)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait_suspend(bar, parity, 20000u)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// ---------------------------------------------------------------------------
// Arithmetic helpers
// ---------------------------------------------------------------------------

// Philox4x32-10 of the counter (quad low, quad high, t, c3).  The counter's
// third word is the step t for every draw of a launch, so round 0's product
// M1 * t is a per-step constant the host supplies (r0_hi_k0 = hi(M1 t) ^ key0,
// r0_lo = lo(M1 t)); rounds 1..9 are the usual ones.
// The 64-bit product a * b as (hi, lo): one wide multiply (measured 0.9%
// faster in the step than the C++ 64-bit product, same bits).
__device__ __forceinline__ void mulwide(uint32_t a, uint32_t b, uint32_t& hi, uint32_t& lo) {
  asm("{\n\t.reg .u64 t;\n\tmul.wide.u32 t, %2, %3;\n\tmov.b64 {%1, %0}, t;\n\t}"
      : "=r"(hi), "=r"(lo) : "r"(a), "r"(b));
}
// The counter's first two words are the 64-bit quad index (qhi, qlo).
__device__ __forceinline__ uint4 philox4x32_10(uint32_t qlo, uint32_t qhi, uint32_t c3,
                                               const StepArgs& a) {
  uint32_t h0, l0;
  mulwide(kPhiloxM0, qlo, h0, l0);
  uint4 c = make_uint4(a.r0_hi_k0 ^ qhi, a.r0_lo, h0 ^ c3 ^ a.rk1[0], l0);
#pragma unroll
  for (int r = 1; r < 10; ++r) {
    uint32_t hi0, lo0, hi1, lo1;
    mulwide(kPhiloxM0, c.x, hi0, lo0);
    mulwide(kPhiloxM1, c.z, hi1, lo1);
    c = make_uint4(hi1 ^ c.y ^ a.rk0[r], lo1, hi0 ^ c.w ^ a.rk1[r], lo0);
  }
  return c;
}

// 1 + u for the draw u in [0,1): the low 23 bits of a word as the mantissa of
// a number in [1, 2).  u = (1 + u) - 1 is exact; u * B rounds like
// fma(1 + u, B, -B).
__device__ __forceinline__ float one_plus_u(uint32_t w) {
  return __uint_as_float((w | 0x3F800000u) & 0x3FFFFFFFu);
}
__device__ __forceinline__ float uniform23(uint32_t w) { return __fsub_rn(one_plus_u(w), 1.0f); }

// The quad index (e0 + off) / 4 of a group at value offset `off` of a block
// starting at element e0, as (low, high) words.  e0 is a multiple of 128 and
// off + 7 < 128, so (e0 / 4) has five zero low bits and adding off / 4 or
// off / 4 + 1 never carries into the high word.
__device__ __forceinline__ uint32_t quad_lo(uint64_t e0, int off) {
  return (uint32_t)(e0 >> 2) + (uint32_t)(off >> 2);
}
__device__ __forceinline__ uint32_t quad_hi(uint64_t e0) { return (uint32_t)(e0 >> 34); }

// The eight draw words of one group: elements 4*quad .. 4*quad + 7.
__device__ __forceinline__ void words8(const StepArgs& a, uint32_t tensor_id, uint32_t stream,
                                       uint32_t qlo, uint32_t qhi, uint32_t r[8]) {
  const uint32_t c3 = tensor_id * 2u + stream;
  const uint4 r0 = philox4x32_10(qlo, qhi, c3, a);
  const uint4 r1 = philox4x32_10(qlo + 1u, qhi, c3, a);
  r[0] = r0.x; r[1] = r0.y; r[2] = r0.z; r[3] = r0.w;
  r[4] = r1.x; r[5] = r1.y; r[6] = r1.z; r[7] = r1.w;
}

__device__ __forceinline__ float bf16lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// binary32 -> bf16, IEEE round to nearest even (the cvt instruction).  Two
// values: lo in bits 0-15, hi in bits 16-31.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint16_t bf16_rn(float x) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float2 f2(float x) { return make_float2(x, x); }

// Three-input maximum and minimum (one instruction each on sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// Largest and smallest |x| over a lane's values (kSub groups of four pairs).
__device__ __forceinline__ float absmax_lane(const float2 (&x)[kSub][4]) {
  float r = fmaxf(fabsf(x[0][0].x), fabsf(x[0][0].y));
#pragma unroll
  for (int s = 0; s < kSub; ++s)
#pragma unroll
    for (int j = (s == 0 ? 1 : 0); j < 4; ++j) r = max3f(r, fabsf(x[s][j].x), fabsf(x[s][j].y));
  return r;
}
__device__ __forceinline__ float absmin_lane(const float2 (&x)[kSub][4]) {
  float r = fminf(fabsf(x[0][0].x), fabsf(x[0][0].y));
#pragma unroll
  for (int s = 0; s < kSub; ++s)
#pragma unroll
    for (int j = (s == 0 ? 1 : 0); j < 4; ++j) r = min3f(r, fabsf(x[s][j].x), fabsf(x[s][j].y));
  return r;
}

// The ZIP-SR uniforms of two draw words: each word rounded to the nearest
// binary32 (ties to even) and scaled by 2^-32, exactly.
__device__ __forceinline__ float2 uniform32x2(uint32_t w0, uint32_t w1, float2 k2m32) {
  return __fmul2_rn(make_float2(__uint2float_rn(w0), __uint2float_rn(w1)), k2m32);
}

// Collectives over the kLanesPerUnit lanes of one block.  FULLW: all lanes
// of the warp execute the call together (every block of the warp takes the
// same path), so it runs with the constant full-warp mask and no convergence
// bookkeeping around it; else with the block's own lane mask `gmask`.
constexpr unsigned kFullMask = 0xFFFFFFFFu;

// Max of non-negative binary32 values over a block's lanes: their bit
// patterns order like the values, so an integer maximum is the exact one.
template <bool FULLW>
__device__ __forceinline__ float unit_max(float v, unsigned gmask) {
  uint32_t b = __float_as_uint(v);
  if (FULLW) {
#pragma unroll
    for (int off = 1; off < kLanesPerUnit; off <<= 1) b = max(b, __shfl_xor_sync(kFullMask, b, off));
    return __uint_as_float(b);
  }
  return __uint_as_float(__reduce_max_sync(gmask, b));
}

// Balanced pairwise sum of (x, y) pairs over a block, from each lane's
// per-group sums: partner offsets 1, 2, 4 join adjacent groups in index order
// within each half of the block, and the two halves (a lane's two groups)
// are joined last.  IEEE addition is commutative, so partners hold the same
// bits.
template <bool FULLW>
__device__ __forceinline__ float2 unit_sum_tree2(const float2 (&v)[kSub], unsigned gmask) {
  const unsigned mask = FULLW ? kFullMask : gmask;
  float2 t[kSub];
#pragma unroll
  for (int s = 0; s < kSub; ++s) t[s] = v[s];
#pragma unroll
  for (int off = 1; off < kLanesPerUnit; off <<= 1) {
#pragma unroll
    for (int s = 0; s < kSub; ++s) {
      const float2 o = make_float2(__shfl_xor_sync(mask, t[s].x, off),
                                   __shfl_xor_sync(mask, t[s].y, off));
      t[s] = __fadd2_rn(t[s], o);
    }
  }
  static_assert(kSub == 2, "the last level joins two halves");
  return __fadd2_rn(t[0], t[1]);
}

// Tables read with data-dependent indices, laid out so that the lanes of a
// warp never meet in a shared-memory bank whatever entries they ask for:
// entry k of each table is one row, and lane c reads its own copy in column
// c of that row.
//   nf4b: NF4 nearest-level buckets {threshold, base code}, one 8-byte copy
//         per half-warp lane (sixteen lanes per wavefront of 8-byte loads);
//   nf4:  NF4 levels, one 4-byte copy per lane;
//   vz:   the zero-inclusive v code points k/15, one copy per lane.
struct LaneTables {
  float2 nf4b[128][16];
  float nf4[16][32];
  float vz[16][32];
};
static __device__ __align__(16) LaneTables g_lane_tables;   // written once per device
__shared__ __align__(16) LaneTables s_lane;                  // each CTA's copy

// Byte offset of the lane's copy of entry (nibble i of `code`) in a table of
// 128-byte rows with 4-byte columns (i is a constant after unrolling, so the
// shift is one instruction and the mask-and-or another).
__device__ __forceinline__ uint32_t nibble_row_off(uint32_t code, int i) {
  const uint32_t t = (4 * i <= 7) ? (code << (7 - 4 * i)) : (code >> (4 * i - 7));
  return (t & 0x780u) | ((threadIdx.x & 31u) << 2);
}
__device__ __forceinline__ float lane_lookup(const float (&tab)[16][32], uint32_t code, int i) {
  return *reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(&tab[0][0]) +
                                         nibble_row_off(code, i));
}

// NF4 nearest level: #{j : x > mid[j]}.  bucket_sum = fma(x, 4096, kMagic +
// 4096) has the bit pattern of kMagic plus r = round(4096 x + 4096), r in
// [0, 8192] for |x| <= 1 + 2^-23, so r & 0x3F80 = 128 floor(r/128) is the
// byte offset of row floor(r/128) of the 128-byte rows, and or-ing in the
// lane's 8-byte column gives the address in one logic operation.  A bucket is
// 1/32 wide in x and holds at most one threshold; there are 128 rows, so any
// masked offset stays inside (rows past 64 read "above all").
__device__ __forceinline__ uint32_t nf4_rtn_bucket(float x, float bucket_sum) {
  const uint32_t off = (__float_as_uint(bucket_sum) & 0x3F80u) | ((threadIdx.x & 15u) << 3);
  const float2 e = *reinterpret_cast<const float2*>(
      reinterpret_cast<const uint8_t*>(&s_lane.nf4b[0][0]) + off);
  return (uint32_t)(__float_as_int(e.y) + (x > e.x ? 1 : 0));
}

// State-space stochastic rounding on the NF4 grid (LM-head m, final 10%).
__device__ __forceinline__ uint32_t nf4_sr(float x, float u, const float* nf4, const float* gap) {
  int j = 0;
#pragma unroll
  for (int i = 1; i <= 14; ++i) j = (nf4[i] <= x) ? i : j;
  const bool lower = __fmul_rn(u, gap[j]) < __fsub_rn(nf4[j + 1], x);
  return lower ? (uint32_t)j : (uint32_t)(j + 1);
}

// Shared tables of one CTA.
struct SmemTables {
  float2 mpair[256];   // byte of two m codes -> their two NF4 levels
  float2 vpair[256];   // byte of two v codes -> their two code points
  float nf4[16];
  float gap[16];
  float vz[16];        // ZIP-SR code points k/15
  float4 zip[16];      // for k0 = nearest integer to 15x: {VZ[k0] (+inf for 15),
                       //   sqrt VZ[k0-1], sqrt VZ[k0], sqrt VZ[k0+1]}
  float2 vzp[16];      // {k/15, (k+1)/15}
  float vzmid[16];     // thresholds between adjacent k/15 code points
};
static_assert(sizeof(SmemTables) % 16 == 0, "tables are copied in 16-byte pieces");

// The shared tables of both code families (0: zero-inclusive v codes, 1:
// zero-excluded), written once per device by the host (cudaMemcpyToSymbol)
// before the first launch; each CTA copies its family's into shared memory.
static __device__ __align__(16) SmemTables g_code_tables[2];

// ---------------------------------------------------------------------------
// Requantisation of one 4-bit block held by kLanesPerUnit lanes (kSub groups
// of 8 values per lane).  FULL: all 128 values valid.  Otherwise myn[s]
// values of group s of this lane are valid.
// ---------------------------------------------------------------------------

// ZIP-SR codes of one group of 8 values, from nv = -v1 and ndv = -d(v1)
// (d = 1/h, the update's denominator) in pairs, and ninv = -1/s of the block.
// FLAT: also test for d(a) == d(b), which needs the state-space fallback;
// callers skip it when the block's R makes that impossible.  U32: the
// binary64 decision of v code 5; else the binary32 one with the whole-word
// uniform.
template <bool FULL, bool FLAT, bool U32>
__device__ __forceinline__ uint32_t zipsr_codes8(const StepArgs& a, const SmemTables& S,
                                                 const float2 (&nv)[4], const float2 (&ndv)[4],
                                                 uint32_t qlo, uint32_t qhi, uint32_t c3,
                                                 float ninv, float R,
                                                 int myn) {
  // two values at a time; from the last pair to the first, so that element i
  // ends in bits 4i..4i+3.  The draws of values 4..7 come from the second
  // Philox call (counter quad + 1), of 0..3 from the first, each made just
  // before its pairs so that only four words are live.
  uint32_t vco = 0;
  uint32_t rw[kGroup];
  if (U32) {   // (the binary64 decision keeps all eight words: fewer live doubles)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint4 r = philox4x32_10(qlo + (uint32_t)c, qhi, c3, a);
      rw[4 * c + 0] = r.x; rw[4 * c + 1] = r.y; rw[4 * c + 2] = r.z; rw[4 * c + 3] = r.w;
    }
  }
#pragma unroll
  for (int j = kGroup / 2 - 1; j >= 0; --j) {
    if (!U32 && (j == 3 || j == 1)) {
      const uint4 r = philox4x32_10(qlo + (uint32_t)(j >> 1), qhi, c3, a);
      rw[4 * (j >> 1) + 0] = r.x; rw[4 * (j >> 1) + 1] = r.y;
      rw[4 * (j >> 1) + 2] = r.z; rw[4 * (j >> 1) + 3] = r.w;
    }
    const float2 x2 = __fmul2_rn(nv[j], f2(ninv));                  // v1 / s
    const float2 t2 = __ffma2_rn(x2, a.k_15, a.k_magic);
    // k0, the nearest integer to 15x, is the bracket or one above it (the top
    // entry's threshold is +inf: its bracket is always 14)
    const uint32_t k0a = __float_as_uint(t2.x) & 15u, k0b = __float_as_uint(t2.y) & 15u;
    const float4 ea = S.zip[k0a], eb = S.zip[k0b];
    const bool deca = x2.x < ea.x, decb = x2.y < eb.x;
    // square roots of the lower and upper code points of each value
    const float2 sa = make_float2(deca ? ea.y : ea.z, decb ? eb.y : eb.z);
    const float2 sb = make_float2(deca ? ea.z : ea.w, decb ? eb.z : eb.w);
    const float2 da = __ffma2_rn(sa, f2(R), a.p_eps);
    const float2 db = __ffma2_rn(sb, f2(R), a.p_eps);
    // fma(y, -1, x) rounds like x - y; nB = -(db - da) dv, rhs = (db - dv) da
    const float2 nB = __fmul2_rn(__ffma2_rn(da, a.k_m1, db), ndv[j]);
    const float2 rhs = __fmul2_rn(__fadd2_rn(db, ndv[j]), da);
    bool lowa, lowb;
    if (U32) {
      // the whole word: (w 2^-32) * B rounded once in binary64, against rhs
      lowa = __dmul_rn((double)rw[2 * j], -(double)nB.x * 0x1p-32) < (double)rhs.x;
      lowb = __dmul_rn((double)rw[2 * j + 1], -(double)nB.y * 0x1p-32) < (double)rhs.y;
    } else {
      // u * B < rhs, with -(u * B) = u * nB rounded once
      const float2 nlhs = __fmul2_rn(uniform32x2(rw[2 * j], rw[2 * j + 1], a.k_2m32), nB);
      lowa = -nlhs.x < rhs.x;
      lowb = -nlhs.y < rhs.y;
    }
    const uint32_t ka = k0a - (deca ? 1u : 0u), kb = k0b - (decb ? 1u : 0u);
    if (FLAT) {
      if (da.x == db.x) {
        const float2 z = S.vzp[ka];
        lowa = U32 ? __dmul_rn((double)rw[2 * j], (double)__fsub_rn(z.y, z.x) * 0x1p-32) <
                         (double)__fsub_rn(z.y, x2.x)
                   : __fmul_rn(__fmul_rn(__uint2float_rn(rw[2 * j]), 0x1p-32f),
                               __fsub_rn(z.y, z.x)) < __fsub_rn(z.y, x2.x);
      }
      if (da.y == db.y) {
        const float2 z = S.vzp[kb];
        lowb = U32 ? __dmul_rn((double)rw[2 * j + 1], (double)__fsub_rn(z.y, z.x) * 0x1p-32) <
                         (double)__fsub_rn(z.y, x2.y)
                   : __fmul_rn(__fmul_rn(__uint2float_rn(rw[2 * j + 1]), 0x1p-32f),
                               __fsub_rn(z.y, z.x)) < __fsub_rn(z.y, x2.y);
      }
    }
    const uint32_t ca = (FULL || 2 * j < myn) ? ka + (lowa ? 0u : 1u) : 0u;
    const uint32_t cb = (FULL || 2 * j + 1 < myn) ? kb + (lowb ? 0u : 1u) : 0u;
    vco = (vco * 16u + cb) * 16u + ca;
  }
  return vco;
}

// The codes k of a pair of zero-excluded values from tm = kMagic + (k + 1),
// k in [0, 15] (exact binary32 integers): tm - 1 is exact, and its bit
// pattern is kMagic's (low byte 0) plus k.  The low byte of the result holds
// k of the first value in bits 0-3 and of the second in bits 4-7.
__device__ __forceinline__ uint32_t ze_code_pair(float2 tm, float2 m1) {
  const float2 kb = __fadd2_rn(tm, m1);                      // m1 = (-1, -1)
  return __float_as_uint(kb.x) + 16u * __float_as_uint(kb.y);
}
// kMagic + max(rint(16x), 1) from t2 = fma(x, 16, kMagic) = kMagic + rint(16x).
__device__ __forceinline__ float2 ze_point(float2 t2) {
  return make_float2(fmaxf(t2.x, kMagic + 1.0f), fmaxf(t2.y, kMagic + 1.0f));
}

// The low bytes of four code pairs as one 32-bit word of eight nibbles
// (value i in bits 4i..4i+3), with the nibbles of values at or past `nvalid`
// cleared.
__device__ __forceinline__ uint32_t pack_code_pairs(const uint32_t (&P)[4], int nvalid) {
  const uint32_t w = __byte_perm(__byte_perm(P[0], P[1], 0x0040), __byte_perm(P[2], P[3], 0x0040),
                                 0x5410);
  return nvalid >= kGroup ? w : w & ((1u << (4 * nvalid)) - 1u);
}

// Value i of a group of eight, held as four pairs.
__device__ __forceinline__ float el(const float2 (&x)[4], int i) {
  return (i & 1) ? x[i >> 1].y : x[i >> 1].x;
}

// RN(1/d) for a block scale d >= FLT_MIN: the fast sequence inside its range,
// else the IEEE division (the branch is uniform over the block's lanes).
__device__ __forceinline__ float block_rcp(float d) {
  if (d >= exact::kRcpLo && d <= exact::kRcpHi) return exact::rcp_rn(d);
  return __fdiv_rn(1.0f, d);
}

// ZIP-SR's R = sqrt(s) rs_bc2 of a block scale s >= FLT_MIN.
__device__ __forceinline__ float zipsr_block_R(const StepArgs& a, float av) {
  const float rs = (av >= exact::kSqrtLo && av <= exact::kSqrtHi) ? exact::sqrt_rn(av)
                                                                   : __fsqrt_rn(av);
  return __fmul_rn(rs, a.rs_bc2);
}
// Whether R rules out two code points of a cell sharing one d value.
__device__ __forceinline__ bool zipsr_not_flat(const StepArgs& a, float R) {
  return R > __fmul_rn(1e-5f, a.eps) && a.eps >= FLT_MIN;
}

// Requantises one block: m1 and nv = -v1 in pairs, ndv = -d(v1) (ZIP-SR),
// am / av = the block's largest |m1| and v1.  Writes this lane's code words
// (group s: word s * kLanesPerUnit + lane of the block's sixteen, from mcb /
// vcb) and, from lane 0, the two scales.
// FAST: the caller has established that am and av lie inside the fast
// sequences' ranges (every |m1| and v1 of the block passed the lanes' range
// checks), that the LM head's stochastic phase does not apply, and for ZIP-SR
// that R = sqrt(av) rs_bc2 (given) rules out flat cells; the code then has no
// branches.  Otherwise each of those is tested here.
template <int VCODE, bool FULL, bool FULLW, bool FAST>
__device__ __forceinline__ void requant_store(const StepArgs& a, const SmemTables& S,
                                              uint32_t tensor_id, uint32_t flags, uint64_t e0,
                                              int lane, const int (&myn)[kSub], unsigned gmask,
                                              const float2 (&m1)[kSub][4],
                                              const float2 (&nv)[kSub][4],
                                              const float2 (&ndv)[kSub][4], float am, float av,
                                              float R_fast, uint32_t* mcb, uint32_t* vcb,
                                              float* msp, float* vsp) {
  // ---- first moment: absmax scale, NF4 codes ----
  uint32_t mco[kSub];
#pragma unroll
  for (int s = 0; s < kSub; ++s) mco[s] = 0;
  float mso = 0.0f;
  if (FAST || am >= FLT_MIN) {
    const float inv = FAST ? exact::rcp_rn(am) : block_rcp(am);
    if (!FAST && (flags & ADAMW4_T_LM_HEAD) && a.lm_sr_active) {
#pragma unroll
      for (int s = 0; s < kSub; ++s) {
        uint32_t rw[kGroup];
        words8(a, tensor_id, kStreamM, quad_lo(e0, group_off(s, lane)), quad_hi(e0), rw);
#pragma unroll
        for (int i = 0; i < kGroup; ++i)
          if (FULL || i < myn[s])
            mco[s] |= nf4_sr(__fmul_rn(el(m1[s], i), inv), uniform23(rw[i]), S.nf4, S.gap)
                      << (4 * i);
      }
    } else {
#pragma unroll
      for (int s = 0; s < kSub; ++s) {
#pragma unroll
        for (int j = kGroup / 2 - 1; j >= 0; --j) {   // last element first
          const float2 x = __fmul2_rn(m1[s][j], f2(inv));
          const float2 b = __ffma2_rn(x, a.k_4096, a.k_magic4096);
          const uint32_t c1 = (FULL || 2 * j + 1 < myn[s]) ? nf4_rtn_bucket(x.y, b.y) : 0u;
          const uint32_t c0 = (FULL || 2 * j < myn[s]) ? nf4_rtn_bucket(x.x, b.x) : 0u;
          mco[s] = (mco[s] * 16u + c1) * 16u + c0;
        }
      }
    }
    mso = am;
  }

  // ---- second moment ----
  uint32_t vco[kSub];
#pragma unroll
  for (int s = 0; s < kSub; ++s) vco[s] = 0;
  float vso = 0.0f;
  if (VCODE == kVZe) {
    // ZE-EDEN ("ZIP-SR / ZE-EDEN", Core equation): nearest zero-excluded
    // code point, scale times ||x||^2 / max(<x,Q(x)>, 1e-12 s^2) on x = v/s.
    // The codes and sums are formed for every block, so that the sums'
    // shuffles run with all the warp's blocks together; an all-zero block
    // (s below FLT_MIN) then stores zeros.
    const bool von = FAST || av >= FLT_MIN;
    // -1/s: x = v1/s is then nv * ninv, the same binary32 product
    const float ninv = FAST ? -exact::rcp_rn(av) : (von ? -block_rcp(av) : 0.0f);
    uint32_t P[kSub][4];
    float2 gsum[kSub];
#pragma unroll
    for (int s = 0; s < kSub; ++s) {
      float2 l1[4];
#pragma unroll
      for (int j = 0; j < kGroup / 2; ++j) {
        const float2 x2 = __fmul2_rn(nv[s][j], f2(ninv));
        const float2 t2 = __ffma2_rn(x2, a.k_16, a.k_magic);       // kMagic + rint(16x)
        const float2 tm = ze_point(t2);                            // kMagic + k + 1
        // (k+1)/16 = tm/16 - kMagic/16: both terms and the result exact
        const float2 q2 = __ffma2_rn(tm, a.k_1_16, a.k_nmagic_16);
        P[s][j] = ze_code_pair(tm, a.k_m1);
        float2 xx = __fmul2_rn(x2, x2);
        float2 xq = __fmul2_rn(x2, q2);
        if (!FULL) {
          if (2 * j >= myn[s]) { xx.x = 0.0f; xq.x = 0.0f; }
          if (2 * j + 1 >= myn[s]) { xx.y = 0.0f; xq.y = 0.0f; }
        }
        // first tree level: (x0^2 + x1^2, x0 q0 + x1 q1), two scalar adds whose
        // results form the pair (cheaper than regrouping the operands)
        l1[j] = make_float2(__fadd_rn(xx.x, xx.y), __fadd_rn(xq.x, xq.y));
      }
      gsum[s] = __fadd2_rn(__fadd2_rn(l1[0], l1[1]), __fadd2_rn(l1[2], l1[3]));
    }
    const float2 t = unit_sum_tree2<FULLW>(gsum, gmask);   // (sum x^2, sum x q)
    if (von) {
#pragma unroll
      for (int s = 0; s < kSub; ++s) vco[s] = pack_code_pairs(P[s], FULL ? kGroup : myn[s]);
      const float den = fmaxf(t.y, 1e-12f);
      // t.x >= 1 - 2^-22 (the block's largest x rounds to 1) and den <= 129:
      // the fast quotient's range holds unless the inputs were not finite
      // (then both forms give a NaN scale)
      const float c = (FAST || (t.x >= 0x1p-60f && t.x <= 0x1p60f && den <= 0x1p60f))
                          ? exact::div_rn(t.x, den)
                          : __fdiv_rn(t.x, den);
      vso = __fmul_rn(av, c);
    }
  } else if (FAST || av >= FLT_MIN) {
    // -1/s: x = v1/s is then nv * ninv, the same binary32 product
    const float ninv = FAST ? -exact::rcp_rn(av) : -block_rcp(av);
    if (VCODE == kVZip || VCODE == kVZip32) {
      // ZIP-SR ("ZIP-SR / ZE-EDEN", Core equation): keep the lower code point
      // with probability [h(v)-h(b)]/[h(a)-h(b)], evaluated division-free as
      // u*((db-da)*dv) < (db-dv)*da with d = 1/h.
      const float R = FAST ? R_fast : zipsr_block_R(a, av);
      const uint32_t c3 = tensor_id * 2u + kStreamV;
      // d(a) == d(b) needs (sqrt(k+1/15) - sqrt(k/15)) R below two ulps of
      // R + eps; the smallest gap is 0.0339, so R > 1e-5 eps rules it out.
      if (FAST || zipsr_not_flat(a, R)) {
#pragma unroll
        for (int s = 0; s < kSub; ++s)
          vco[s] = zipsr_codes8<FULL, false, VCODE == kVZip32>(
              a, S, nv[s], ndv[s], quad_lo(e0, group_off(s, lane)), quad_hi(e0), c3, ninv, R,
              myn[s]);
      } else {
#pragma unroll
        for (int s = 0; s < kSub; ++s)
          vco[s] = zipsr_codes8<FULL, true, VCODE == kVZip32>(
              a, S, nv[s], ndv[s], quad_lo(e0, group_off(s, lane)), quad_hi(e0), c3, ninv, R,
              myn[s]);
      }
      vso = av;
    } else if (VCODE == kVZiRtn || VCODE == kVZiSr) {
      // State-space rules on the zero-inclusive code: nearest code point, or
      // the lower one with probability (b - x)/(b - a).
#pragma unroll
      for (int s = 0; s < kSub; ++s) {
        uint32_t rw[kGroup];
        if (VCODE == kVZiSr)
          words8(a, tensor_id, kStreamV, quad_lo(e0, group_off(s, lane)), quad_hi(e0), rw);
#pragma unroll
        for (int j = kGroup / 2 - 1; j >= 0; --j) {   // last element first
          const float2 x2 = __fmul2_rn(nv[s][j], f2(ninv));
          const float2 t2 = __ffma2_rn(x2, a.k_15, a.k_magic);
#pragma unroll
          for (int h = 1; h >= 0; --h) {
            const int i = 2 * j + h;
            const float x = h ? x2.y : x2.x;
            const uint32_t k0 = __float_as_uint(h ? t2.y : t2.x) & 15u;
            const uint32_t k = k0 - ((x < S.zip[k0].x) ? 1u : 0u);   // the bracket
            uint32_t c;
            if (VCODE == kVZiRtn) {
              c = k + ((x > S.vzmid[k]) ? 1u : 0u);
            } else {
              const float2 z = S.vzp[k];
              const bool lower =
                  __fmul_rn(uniform23(rw[i]), __fsub_rn(z.y, z.x)) < __fsub_rn(z.y, x);
              c = k + (lower ? 0u : 1u);
            }
            vco[s] = vco[s] * 16u + ((FULL || i < myn[s]) ? c : 0u);
          }
        }
      }
      vso = av;
    } else if (VCODE == kVZeFloor) {
      // Zero-excluded code with a positive floor: nearest (k+1)/16, no rescale.
#pragma unroll
      for (int s = 0; s < kSub; ++s) {
        uint32_t P[4];
#pragma unroll
        for (int j = 0; j < kGroup / 2; ++j) {
          const float2 x2 = __fmul2_rn(nv[s][j], f2(ninv));
          const float2 t2 = __ffma2_rn(x2, a.k_16, a.k_magic);       // kMagic + rint(16x)
          P[j] = ze_code_pair(ze_point(t2), a.k_m1);
        }
        vco[s] = pack_code_pairs(P, FULL ? kGroup : myn[s]);
      }
      vso = av;
    }
  }

#pragma unroll
  for (int s = 0; s < kSub; ++s) {
    mcb[s * kLanesPerUnit + lane] = mco[s];
    vcb[s * kLanesPerUnit + lane] = vco[s];
  }
  if (lane == 0) {
    *msp = mso;
    *vsp = vso;
  }
}

// How a group's codes are decoded, chosen per v code by measurement.  The
// lane tables (one 4-byte load per value, no bank conflicts, two more
// instructions per value for the address) pay for the zero-inclusive codes;
// the zero-excluded ones decode v by arithmetic and keep the pair table for
// m (one 8-byte load per two values), which costs them fewer instructions.
constexpr int kVDecPair = 0;      // v through the pair table
constexpr int kVDecZeArith = 1;   // v = (k + 1)/16 by arithmetic (zero-excluded)
constexpr int kVDecLaneVz = 2;    // v through the lane table of k/15 (zero-inclusive)
template <int VCODE>
__host__ __device__ constexpr bool zero_excluded() {
  return VCODE == kVZe || VCODE == kVZeFloor;
}
template <int VCODE>
__host__ __device__ constexpr int v_decode() {
  return zero_excluded<VCODE>() ? kVDecZeArith : kVDecLaneVz;
}
template <int VCODE>
__host__ __device__ constexpr bool m_lane_decode() {
  return !zero_excluded<VCODE>();
}

// Decode and moment update for one group of 8 values of a 4-bit block
// ("ZIP-SR / ZE-EDEN", Method flowchart: decode the prior moments, update
// them).  Out: m1 and nv = -v1 in pairs.  VDEC: how the v codes are decoded;
// MLANE: the m codes through the lane table.
template <int VDEC, bool MLANE>
__device__ __forceinline__ void moments8(const StepArgs& a, const SmemTables& S,
                                         const float (&g)[kGroup], uint32_t mc, uint32_t vc,
                                         float2 sm, float2 sv, float2 (&m1)[4], float2 (&nv)[4]) {
#pragma unroll
  for (int j = 0; j < kGroup / 2; ++j) {
    // one byte holds the codes of values 2j (low nibble) and 2j+1 (high nibble)
    const float2 mq = MLANE ? make_float2(lane_lookup(s_lane.nf4, mc, 2 * j),
                                                 lane_lookup(s_lane.nf4, mc, 2 * j + 1))
                                   : S.mpair[__byte_perm(mc, 0, 0x4440 + j)];
    const float2 m0 = __fmul2_rn(mq, sm);
    float2 vq;
    if (VDEC == kVDecZeArith) {
      // The two nibbles of byte j, left in place in the low 16 bits of the
      // word (bytes 2 and 3 shifted down first), or-ed into kMagic's
      // mantissa: kMagic + k 2^p, exact, with p = 8 (j & 1) or 8 (j & 1) + 4.
      // Then (k + 1)/16 = (kMagic + k 2^p) 2^-(p+4) + (1/16 - kMagic 2^-(p+4)),
      // one fma whose product, addend and result are all exact.
      const uint32_t w = (j < 2) ? vc : (vc >> 16);
      const uint32_t lo = (w & (0x0Fu << (8 * (j & 1)))) | 0x4B400000u;
      const uint32_t hi = (w & (0xF0u << (8 * (j & 1)))) | 0x4B400000u;
      vq = __ffma2_rn(make_float2(__uint_as_float(lo), __uint_as_float(hi)),
                      (j & 1) ? a.k_ze_scale1 : a.k_ze_scale0,
                      (j & 1) ? a.k_ze_off1 : a.k_ze_off0);
    } else if (VDEC == kVDecLaneVz) {
      vq = make_float2(lane_lookup(s_lane.vz, vc, 2 * j), lane_lookup(s_lane.vz, vc, 2 * j + 1));
    } else {
      vq = S.vpair[__byte_perm(vc, 0, 0x4440 + j)];
    }
    const float2 v0 = __fmul2_rn(vq, sv);
    const float2 gg = make_float2(g[2 * j], g[2 * j + 1]);
    m1[j] = __ffma2_rn(a.p_b1, m0, __fmul2_rn(a.p_omb1, gg));
    // -v1 = fma(-b2, v0, -(1-b2) g^2), the negation of the canonical v1 exactly
    nv[j] = __ffma2_rn(a.p_nb2, v0, __fmul2_rn(a.p_nomb2, __fmul2_rn(gg, gg)));
  }
}

// Whether all a lane's |m1| and v1 lie in the fast sequences' ranges (also
// true of the block scales then: am in [2^-60, 2^100], av in [2^-100, 2^64]).
// lam / lav: the lane's largest |m1| and v1.
__device__ __forceinline__ bool lane_in_range(const StepArgs& a, const float2 (&m1)[kSub][4],
                                              const float2 (&nv)[kSub][4], float lam, float lav) {
  return absmin_lane(m1) >= a.m_lo && lam <= a.m_hi && absmin_lane(nv) >= a.v_lo &&
         lav <= a.v_hi;
}

// Weight update of a group of 8 values from their working moments ("ZIP-SR /
// ZE-EDEN", Core equation: the weights use the unquantised moments): the
// square root and the division from exact_math.cuh (operands in range), in
// pairs.  Out: ndv = -d(v1) (KEEP_DV), nfacc += 0 * w.
template <bool KEEP_DV>
__device__ __forceinline__ void weights8_fast(const StepArgs& a, float decay, float (&w)[kGroup],
                                              const float2 (&m1)[4], const float2 (&nv)[4],
                                              float2 (&ndv)[4], float2& nfacc) {
#pragma unroll
  for (int j = 0; j < kGroup / 2; ++j) {
    const float2 ns = exact::neg_sqrt2_rn(nv[j], a.k_half);         // -sqrt(v1)
    const float2 nd = __ffma2_rn(ns, a.p_rs, a.p_neps);             // -(sqrt(v1) rs + eps)
    const float2 q = exact::div2_rn_neg(m1[j], nd, a.k_one);        // m1 / den
    const float2 ww = __ffma2_rn(a.p_nstep, q,
                                 __fmul2_rn(make_float2(w[2 * j], w[2 * j + 1]), f2(decay)));
    if (KEEP_DV) ndv[j] = nd;
    w[2 * j] = ww.x;
    w[2 * j + 1] = ww.y;
    nfacc = __ffma2_rn(ww, a.k_zero, nfacc);
  }
}

// The same with the IEEE operations, value by value (FULL false: the first
// `myn` values only).
template <bool FULL, bool KEEP_DV>
__device__ __forceinline__ void weights8_ieee(const StepArgs& a, float decay, float (&w)[kGroup],
                                              const float2 (&m1)[4], const float2 (&nv)[4],
                                              float2 (&ndv)[4], int myn, float2& nfacc) {
#pragma unroll
  for (int i = 0; i < kGroup; ++i) {
    if (FULL || i < myn) {
      const float v1 = -el(nv, i);
      const float den = __fmaf_rn(__fsqrt_rn(v1), a.rs_bc2, a.eps);
      const float wi = __fmaf_rn(a.nstep, __fdiv_rn(el(m1, i), den), __fmul_rn(w[i], decay));
      w[i] = wi;
      if (KEEP_DV) {
        if (i & 1) ndv[i >> 1].y = -den;
        else ndv[i >> 1].x = -den;
      }
      nfacc.x = __fmaf_rn(wi, 0.0f, nfacc.x);
    }
  }
}

// Weight i of a group, fp32 or (BF16W and flagged) bf16.
template <bool BF16W>
__device__ __forceinline__ float load_w(const float* wp, const uint16_t* wp16, bool wbf, int i) {
  if (BF16W && wbf) return __uint_as_float((uint32_t)wp16[i] << 16);
  return wp[i];
}
template <bool BF16W>
__device__ __forceinline__ void store_w(float* wp, uint16_t* wp16, bool wbf, int i, float x) {
  if (BF16W && wbf) wp16[i] = bf16_rn(x);
  else wp[i] = x;
}

// A unit read straight from global memory: a ragged last 4-bit block or a
// chunk of an fp32-state tensor.  Both take the IEEE operations value by
// value.
template <int VCODE, bool BF16W>
__device__ __forceinline__ void process_direct(const StepArgs& a, const SmemTables& S,
                                               const StateArena& st, const UnitHeader* hdp,
                                               int lane, unsigned gmask, float2& nfacc) {
  const int nval = (int)(hdp->nv_soff & 255u);
  const uint32_t flags = hdp->flags;
  const bool wbf = BF16W && (flags & kBf16W);
  const float decay = hdp->decay;
  int myn[kSub];
  float w[kSub][kGroup], g[kSub][kGroup];
#pragma unroll
  for (int s = 0; s < kSub; ++s) {
    const int o = group_off(s, lane);
    myn[s] = min(max(nval - o, 0), kGroup);
    // the header's w is the unit's first weight, of either width
    const float* wp = wbf ? nullptr : hdp->w + o;
    const uint16_t* wp16 = wbf ? reinterpret_cast<const uint16_t*>(hdp->w) + o : nullptr;
    const uint16_t* gp = hdp->g + o;
#pragma unroll
    for (int i = 0; i < kGroup; ++i) {
      w[s][i] = (i < myn[s]) ? load_w<BF16W>(wp, wp16, wbf, i) : 0.0f;
      g[s][i] = (i < myn[s]) ? __uint_as_float((uint32_t)gp[i] << 16) : 0.0f;
    }
  }
  if (flags & kKindFp32) {
#pragma unroll
    for (int s = 0; s < kSub; ++s) {
      const int o = group_off(s, lane);
      float* wp = wbf ? nullptr : hdp->w + o;
      uint16_t* wp16 = wbf ? reinterpret_cast<uint16_t*>(hdp->w) + o : nullptr;
      float* mp = reinterpret_cast<float*>(hdp->mc) + o;
      float* vp = reinterpret_cast<float*>(hdp->vc) + o;
#pragma unroll
      for (int i = 0; i < kGroup; ++i) {
        if (i < myn[s]) {
          const float gi = g[s][i];
          const float m1 = __fmaf_rn(a.b1, mp[i], __fmul_rn(a.omb1, gi));
          const float v1 = __fmaf_rn(a.b2, vp[i], __fmul_rn(a.omb2, __fmul_rn(gi, gi)));
          const float den = __fmaf_rn(__fsqrt_rn(v1), a.rs_bc2, a.eps);
          const float wi = __fmaf_rn(-a.step_size, __fdiv_rn(m1, den), __fmul_rn(w[s][i], decay));
          store_w<BF16W>(wp, wp16, wbf, i, wi);
          nfacc.x = __fmaf_rn(wi, 0.0f, nfacc.x);
          mp[i] = m1;
          vp[i] = v1;
        }
      }
    }
    return;
  }
  // a ragged last block of a 4-bit tensor
  constexpr bool kKeepDv = (VCODE == kVZip || VCODE == kVZip32);
  float* msp = hdp->ms;
  float* vsp = msp + st.vs_minus_ms;
  const float2 sm = f2(*msp), sv = f2(*vsp);
  float2 m1[kSub][4], nv[kSub][4], ndv[kSub][4];
  float lam = 0.0f, lav = 0.0f;
#pragma unroll
  for (int s = 0; s < kSub; ++s) {
    moments8<v_decode<VCODE>(), m_lane_decode<VCODE>()>(a, S, g[s], hdp->mc[s * kLanesPerUnit + lane],
                       hdp->vc[s * kLanesPerUnit + lane], sm,
             sv, m1[s], nv[s]);
#pragma unroll
    for (int j = 0; j < kGroup / 2; ++j) ndv[s][j] = f2(-1.0f);   // (slots past myn)
#pragma unroll
    for (int i = 0; i < kGroup; ++i) {
      if (i < myn[s]) {
        lam = fmaxf(lam, fabsf(el(m1[s], i)));
        lav = fmaxf(lav, fabsf(el(nv[s], i)));
      }
    }
    weights8_ieee<false, kKeepDv>(a, decay, w[s], m1[s], nv[s], ndv[s], myn[s], nfacc);
    const int o = group_off(s, lane);
    float* wp = wbf ? nullptr : hdp->w + o;
    uint16_t* wp16 = wbf ? reinterpret_cast<uint16_t*>(hdp->w) + o : nullptr;
#pragma unroll
    for (int i = 0; i < kGroup; ++i)
      if (i < myn[s]) store_w<BF16W>(wp, wp16, wbf, i, w[s][i]);
  }
  const float am = unit_max<false>(lam, gmask);
  const float av = unit_max<false>(lav, gmask);
  requant_store<VCODE, false, false, false>(a, S, hdp->tensor_id, flags, hdp->e0, lane, myn, gmask,
                                            m1, nv, ndv, am, av, 0.0f, hdp->mc, hdp->vc, msp, vsp);
}

// A tensor descriptor read with four 16-byte loads.
__device__ __forceinline__ DevTensor load_tensor(const DevTensor* p) {
  DevTensor d;
  const uint4* src = reinterpret_cast<const uint4*>(p);
  uint4* dst = reinterpret_cast<uint4*>(&d);
#pragma unroll
  for (int i = 0; i < (int)(sizeof(DevTensor) / 16); ++i) dst[i] = __ldg(src + i);
  return d;
}

// ---------------------------------------------------------------------------
// Producer: fills CTA-wide stages, one tile of kTileUnits consecutive units
// each.  Lane i handles unit i of the tile (header, scales); the lane that
// starts a run of whole 4-bit blocks of one tensor issues that run's bulk
// copies.
// ---------------------------------------------------------------------------
template <bool BF16W>
__device__ __forceinline__ void produce(const DevTensor* __restrict__ T, int64_t u_begin,
                                        int64_t u_end, const StepArgs& a, const StateArena& st,
                                        uint8_t* stages, uint32_t full0, uint32_t empty0,
                                        int lane) {
  constexpr unsigned kMask = kTileUnits == 32 ? kFullMask : (1u << kTileUnits) - 1u;
  const int64_t ntiles = (u_end - u_begin + kTileUnits - 1) / kTileUnits;
  int ti = -1;
  int64_t t_begin = 0, t_end = 0, t_numel = 0, t_soff = 0, t_eoff = 0;
  float* t_param = nullptr;
  const uint16_t* t_grad = nullptr;
  uint32_t t_id = 0, t_flags = 0;
  float t_decay = 1.0f;
  const uint32_t stages_s = smem_addr(stages);
  int s = 0;
  uint32_t round = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const uint32_t full = full0 + 8u * s;
    if (round > 0 && !__all_sync(kMask, wait_phase_suspended(empty0 + 8u * s, (round - 1) & 1u,
                                                           kWaitLimitNs))) {
      // Leaving early: flag it, then wait (bounded) for the copies this warp
      // issued into stages not yet handed back.  Stage j was last filled in
      // this round if j < s, else in the previous one; its full barrier
      // completes that fill's phase once the bytes have landed.
      if (lane == 0) atomicOr(a.status, 1u);
      for (int j = 0; j < kStages; ++j) {
        const uint32_t last = (j < s) ? round : round - 1;
        wait_phase_suspended(full0 + 8u * j, last & 1u, kDrainLimitNs);
      }
      cp_async_wait_all();
      return;
    }
    const int64_t u = u_begin + tile * kTileUnits + lane;
    bool has = u < u_end;
    if (has && u >= t_end) {
      DevTensor d;
      do {
        d = load_tensor(&T[++ti]);    // the whole descriptor in one round trip
      } while (u >= d.unit_end);
      t_end = d.unit_end;
      t_begin = d.unit_begin;
      t_numel = d.numel;
      t_soff = d.state_off;
      t_eoff = (int64_t)d.block_offset * kBlock;
      t_param = d.param;
      t_grad = d.grad;
      t_id = d.tensor_id;
      t_flags = d.flags;
      t_decay = (float)(1.0 - (double)a.lr * (double)d.weight_decay);
    }
    const int64_t ub = u - t_begin;
    const int64_t e0 = ub * kBlock;
#ifdef ADAMW4_CHECKED
    // Checked build: the unit's values lie inside its tensor and its state
    // inside the arena; otherwise the status word gets bit 1 and the unit is
    // dropped (no copy, no consumer work).
    if (has) {
      const int64_t nv = min((int64_t)kBlock, t_numel - e0);
      const bool ok = ub >= 0 && nv > 0 && u < t_end &&
                      ((t_flags & kKindFp32) ? (t_soff >= 0 && t_soff + e0 + nv <= st.n32)
                                             : (t_soff >= 0 && t_soff + ub < st.nblocks4));
      if (!ok) {
        atomicOr(a.status, 2u);
        has = false;
      }
    }
#endif
    const int nvalid = has ? (int)min((int64_t)kBlock, t_numel - e0) : 0;
    const bool staged = has && !(t_flags & kKindFp32) && nvalid == kBlock;
    const bool wbf = BF16W && (t_flags & kBf16W);       // bf16 weights: 256 B per unit
    uint8_t* sp = stages + s * kStageBytes;
    UnitHeader* hd = reinterpret_cast<UnitHeader*>(sp + kOffHdr) + lane;
    hd->w = wbf ? reinterpret_cast<float*>(reinterpret_cast<uint16_t*>(t_param) + e0)
                : t_param + e0;
    hd->g = t_grad + e0;
    hd->e0 = (uint64_t)(t_eoff + e0);   // keys the draws
    if (t_flags & kKindFp32) {
      hd->mc = reinterpret_cast<uint32_t*>(st.fm + t_soff + e0);
      hd->vc = reinterpret_cast<uint32_t*>(st.fv + t_soff + e0);
      hd->ms = nullptr;
    } else {
      const int64_t blk = t_soff + ub;
      hd->mc = reinterpret_cast<uint32_t*>(st.mcodes + blk * (kBlock / 2));
      hd->vc = reinterpret_cast<uint32_t*>(st.vcodes + blk * (kBlock / 2));
      hd->ms = st.mscale + blk;
    }
    hd->tensor_id = t_id;
    hd->flags = has ? (t_flags | (staged ? kStaged : 0u)) : kNoUnit;
    hd->decay = t_decay;
    // Runs of whole blocks of one tensor are contiguous in global memory and
    // in the stage: one bulk copy per array per run.
    const unsigned staged_mask = __ballot_sync(kMask, staged);
    const int prev_ti = __shfl_up_sync(kMask, ti, 1);
    const bool cont = staged && lane > 0 && ((staged_mask >> (lane - 1)) & 1u) && prev_ti == ti;
    const unsigned cont_mask = __ballot_sync(kMask, cont);
    const uint32_t dst = stages_s + (uint32_t)(s * kStageBytes);
    uint32_t tx = (uint32_t)__popc(staged_mask) * kUnitTx;
    if (BF16W) tx -= (uint32_t)__popc(__ballot_sync(kMask, staged && wbf)) * 256u;
    uint32_t w_soff = 0;
    if (BF16W) {
      // A run's weights land packed at the start of its own units' 512-B w
      // slots: 512 B per unit for fp32, 256 B for bf16.  The run starts at the
      // nearest lane at or below this one that does not continue a run
      // ((2 << 31) - 1 wraps to the full mask).
      const int start = 31 - __clz(~cont_mask & ((2u << lane) - 1u));
      w_soff = (uint32_t)(kOffW + start * 512 + (lane - start) * (wbf ? 256 : 512));
    }
    hd->nv_soff = (uint32_t)nvalid | (w_soff << 8);
    // Publish the headers: the warp barrier orders every lane's header stores
    // before lane 0's arrive, whose release (mbarrier.arrive is a release at
    // CTA scope) the consumers' acquiring wait on the phase then covers.
    __syncwarp(kMask);
    if (lane == 0) mbar_arrive_expect_tx(full, tx);
    if (staged && !cont && !a.fault_stall) {
      // this lane starts a run: it extends over the following lanes whose
      // unit continues it (the shift is done in 64 bits: lane + 1 may be 32)
      const unsigned rest = ~(uint32_t)((uint64_t)cont_mask >> (lane + 1));
      const int len = __ffs(rest);          // 1 + number of continuing lanes
      const int64_t blk = t_soff + ub;
      if (wbf)
        bulk_g2s(dst + kOffW + lane * 512, reinterpret_cast<const uint16_t*>(t_param) + e0,
                 256u * len, full);
      else
        bulk_g2s(dst + kOffW + lane * 512, t_param + e0, 512u * len, full);
      bulk_g2s(dst + kOffG + lane * 256, t_grad + e0, 256u * len, full);
      bulk_g2s(dst + kOffMC + lane * 64, st.mcodes + blk * (kBlock / 2), 64u * len, full);
      bulk_g2s(dst + kOffVC + lane * 64, st.vcodes + blk * (kBlock / 2), 64u * len, full);
    }
    if (staged && !a.fault_stall) {
      const int64_t blk = t_soff + ub;
      cp_async4(dst + kOffMS + lane * 8, st.mscale + blk);
      cp_async4(dst + kOffMS + lane * 8 + 4, st.mscale + blk);
      cp_async4(dst + kOffVS + lane * 8, st.vscale + blk);
      cp_async4(dst + kOffVS + lane * 8 + 4, st.vscale + blk);
    }
    cp_async_arrive_noinc(full);            // one arrival per lane, when its copies land
    // (test hook: with the stall armed no bulk copy is issued, so the expected
    // bytes never arrive and the consumers' waits run out)
    if (++s == kStages) {
      s = 0;
      ++round;
    }
  }
  cp_async_wait_all();
}

// Stores one group of a lane's updated weights (value offset `off` in the
// block; 16-byte stores): fp32, or (wbf) bf16 rounded to nearest even.
template <bool BF16W>
__device__ __forceinline__ void store_w8(float* w0, bool wbf, int off, const float (&w)[kGroup]) {
  if (BF16W && wbf) {
    uint16_t* wp = reinterpret_cast<uint16_t*>(w0) + off;
    *reinterpret_cast<uint4*>(wp) = make_uint4(bf16x2_rn(w[0], w[1]), bf16x2_rn(w[2], w[3]),
                                               bf16x2_rn(w[4], w[5]), bf16x2_rn(w[6], w[7]));
  } else {
    float* wp = w0 + off;
    *reinterpret_cast<float4*>(wp) = make_float4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<float4*>(wp + 4) = make_float4(w[4], w[5], w[6], w[7]);
  }
}

// A whole 4-bit block whose data is in the stage, slot `unit` of the tile.
// FULLW: all the warp's blocks take this path together (see unit_max).  Then,
// when every lane of every such block has its moments inside the fast ranges
// (and no block is an LM head in its stochastic phase, nor, for ZIP-SR,
// flat), the blocks run one branch-free sequence; a warp that does not
// qualify takes the general sequence, with its per-lane and per-block range
// tests.
template <int VCODE, bool BF16W, bool FULLW>
__device__ __forceinline__ void process_staged(const StepArgs& a, const SmemTables& S,
                                               const StateArena& st, const uint8_t* sp,
                                               const UnitHeader* hdp, uint32_t flags, int unit,
                                               int lane, unsigned gmask, float2& nfacc) {
  constexpr bool kKeepDv = (VCODE == kVZip || VCODE == kVZip32);
  constexpr bool kZip = (VCODE == kVZip || VCODE == kVZip32);
  float w[kSub][kGroup], g[kSub][kGroup];
  uint32_t mc[kSub], vc[kSub];
  const bool wbf = BF16W && (flags & kBf16W);
#pragma unroll
  for (int s = 0; s < kSub; ++s) {
    const int o = group_off(s, lane);
    const uint4 gg = *reinterpret_cast<const uint4*>(sp + kOffG + unit * 256 + o * 2);
    if (wbf) {
      const uint4 wr = *reinterpret_cast<const uint4*>(sp + (hdp->nv_soff >> 8) + o * 2);
      w[s][0] = bf16lo(wr.x); w[s][1] = bf16hi(wr.x); w[s][2] = bf16lo(wr.y);
      w[s][3] = bf16hi(wr.y); w[s][4] = bf16lo(wr.z); w[s][5] = bf16hi(wr.z);
      w[s][6] = bf16lo(wr.w); w[s][7] = bf16hi(wr.w);
    } else {
      const uint8_t* wsrc = sp + kOffW + unit * 512 + o * 4;
      const float4 wa = *reinterpret_cast<const float4*>(wsrc);
      const float4 wb = *reinterpret_cast<const float4*>(wsrc + 16);
      w[s][0] = wa.x; w[s][1] = wa.y; w[s][2] = wa.z; w[s][3] = wa.w;
      w[s][4] = wb.x; w[s][5] = wb.y; w[s][6] = wb.z; w[s][7] = wb.w;
    }
    g[s][0] = bf16lo(gg.x); g[s][1] = bf16hi(gg.x); g[s][2] = bf16lo(gg.y);
    g[s][3] = bf16hi(gg.y); g[s][4] = bf16lo(gg.z); g[s][5] = bf16hi(gg.z);
    g[s][6] = bf16lo(gg.w); g[s][7] = bf16hi(gg.w);
    mc[s] = *reinterpret_cast<const uint32_t*>(sp + kOffMC + unit * 64 + o / 2);
    vc[s] = *reinterpret_cast<const uint32_t*>(sp + kOffVC + unit * 64 + o / 2);
  }
  const float2 sm = *reinterpret_cast<const float2*>(sp + kOffMS + unit * 8);
  const float2 sv = *reinterpret_cast<const float2*>(sp + kOffVS + unit * 8);
  const float decay = hdp->decay;

  float2 m1[kSub][4], nv[kSub][4], ndv[kSub][4];
#pragma unroll
  for (int s = 0; s < kSub; ++s)
    moments8<v_decode<VCODE>(), m_lane_decode<VCODE>()>(a, S, g[s], mc[s], vc[s], sm, sv, m1[s], nv[s]);
  const float lam = absmax_lane(m1);
  const float lav = absmax_lane(nv);
  const float am = unit_max<FULLW>(lam, gmask);
  const float av = unit_max<FULLW>(lav, gmask);
  const bool lane_fast = lane_in_range(a, m1, nv, lam, lav);
  bool warp_fast = false;
  float R = 0.0f;
  if (FULLW) {
    bool ok = lane_fast && !((flags & ADAMW4_T_LM_HEAD) && a.lm_sr_active);
    if (kZip) {
      R = __fmul_rn(exact::sqrt_rn(av), a.rs_bc2);   // av in range whenever `ok` holds
      ok = ok && zipsr_not_flat(a, R);
    }
    warp_fast = __all_sync(kFullMask, ok);
  }
  int nall[kSub];
#pragma unroll
  for (int s = 0; s < kSub; ++s) nall[s] = kGroup;
  float* msp = hdp->ms;
  if (warp_fast) {
#pragma unroll
    for (int s = 0; s < kSub; ++s) {
      weights8_fast<kKeepDv>(a, decay, w[s], m1[s], nv[s], ndv[s], nfacc);
      store_w8<BF16W>(hdp->w, wbf, group_off(s, lane), w[s]);
    }
    requant_store<VCODE, true, FULLW, true>(a, S, hdp->tensor_id, flags, hdp->e0, lane, nall,
                                            gmask, m1, nv, ndv, am, av, R, hdp->mc, hdp->vc, msp,
                                            msp + st.vs_minus_ms);
  } else {
#pragma unroll
    for (int s = 0; s < kSub; ++s) {
      if (lane_fast) weights8_fast<kKeepDv>(a, decay, w[s], m1[s], nv[s], ndv[s], nfacc);
      else weights8_ieee<true, kKeepDv>(a, decay, w[s], m1[s], nv[s], ndv[s], kGroup, nfacc);
      store_w8<BF16W>(hdp->w, wbf, group_off(s, lane), w[s]);
    }
    requant_store<VCODE, true, FULLW, false>(a, S, hdp->tensor_id, flags, hdp->e0, lane, nall,
                                             gmask, m1, nv, ndv, am, av, 0.0f, hdp->mc, hdp->vc,
                                             msp, msp + st.vs_minus_ms);
  }
}

// ---------------------------------------------------------------------------
// The step kernel
// ---------------------------------------------------------------------------

template <int VCODE, bool BF16W>
__global__ void __launch_bounds__(kCtaThreads, kMinCtasPerSm)
adamw4_step_kernel(const DevTensor* __restrict__ T, int64_t u_begin, int64_t u_end, StepArgs a,
                   StateArena st) {
  extern __shared__ __align__(128) uint8_t s_stage[];
  __shared__ __align__(8) uint64_t s_full[kStages];
  __shared__ __align__(8) uint64_t s_empty[kStages];
  __shared__ SmemTables S;

  if (threadIdx.x < kStages) {
    // full: the producer's expect-tx arrive plus one cp.async arrive per
    // producer lane; empty: one release per unit slot
    mbar_init(smem_addr(&s_full[threadIdx.x]), 1 + kTileUnits);
    mbar_init(smem_addr(&s_empty[threadIdx.x]), kTileUnits);
    fence_mbar_init();
  }
  __syncthreads();

  const uint32_t full0 = smem_addr(&s_full[0]);
  const uint32_t empty0 = smem_addr(&s_empty[0]);
  const int warp = threadIdx.x >> 5;
  if (warp == kProducerWarp) {
    // (starts on the first tile at once; the tables are the consumers' concern)
    const int lane = threadIdx.x & 31;
    if (lane < kTileUnits) produce<BF16W>(T, u_begin, u_end, a, st, s_stage, full0, empty0, lane);
    return;
  }

  // The consumers copy their code family's tables and the lane tables into
  // shared memory while the producer fetches the first tiles, then meet at
  // barrier 1 (consumer threads only; barrier 0 is the CTA-wide one above).
  {
    constexpr int kFamily = (VCODE == kVZe || VCODE == kVZeFloor) ? 1 : 0;   // zero-excluded
    constexpr int kT = (int)(sizeof(SmemTables) / 16);
    constexpr int kAll = kT + (int)(sizeof(LaneTables) / 16);
    constexpr int kPerThread = (kAll + kConsumerThreads - 1) / kConsumerThreads;
    const uint4* srcT = reinterpret_cast<const uint4*>(&g_code_tables[kFamily]);
    const uint4* srcB = reinterpret_cast<const uint4*>(&g_lane_tables);
    uint4* dstT = reinterpret_cast<uint4*>(&S);
    uint4* dstB = reinterpret_cast<uint4*>(&s_lane);
    uint4 r[kPerThread];   // every load issued before the first store: one round trip
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int i = threadIdx.x + k * kConsumerThreads;
      if (i < kAll) r[k] = __ldg(i < kT ? srcT + i : srcB + (i - kT));
    }
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int i = threadIdx.x + k * kConsumerThreads;
      if (i < kT) dstT[i] = r[k];
      else if (i < kAll) dstB[i - kT] = r[k];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");
  }

  // ---- consumers: the kLanesPerUnit lanes of slot `unit` take unit `unit`
  // of every tile ----
  const int lane = threadIdx.x & (kLanesPerUnit - 1);
  const int unit = threadIdx.x / kLanesPerUnit;
  const unsigned gmask = ((1u << kLanesPerUnit) - 1u) << (threadIdx.x & 31 & ~(kLanesPerUnit - 1));
  const int64_t ntiles = (u_end - u_begin + kTileUnits - 1) / kTileUnits;
  int s = 0;
  uint32_t parity = 0;
  float2 nfacc = make_float2(0.0f, 0.0f);   // NaN once an updated weight is not finite
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const uint32_t full = full0 + 8u * s;
    const uint32_t empty = empty0 + 8u * s;
    if (!__all_sync(kFullMask, wait_phase(full, parity, kWaitLimitNs))) {
      if ((threadIdx.x & 31) == 0) atomicOr(a.status, 1u);
      return;
    }
    const uint8_t* sp = s_stage + s * kStageBytes;
    const UnitHeader* hdp = reinterpret_cast<const UnitHeader*>(sp + kOffHdr) + unit;
    const uint32_t flags = hdp->flags;
    const bool staged = (flags & kStaged) != 0;
    if (__all_sync(kFullMask, staged)) {          // every block of the warp is whole and staged
      process_staged<VCODE, BF16W, true>(a, S, st, sp, hdp, flags, unit, lane, gmask, nfacc);
    } else if (staged) {
      process_staged<VCODE, BF16W, false>(a, S, st, sp, hdp, flags, unit, lane, gmask, nfacc);
    } else if (!(flags & kNoUnit)) {
      process_direct<VCODE, BF16W>(a, S, st, hdp, lane, gmask, nfacc);
    }
    // every read of the stage (header included) is done: hand it back, one
    // arrival per unit slot (all of the warp's, from its lane 0)
    fence_proxy_async_smem();
    __syncwarp(kFullMask);
    if ((threadIdx.x & 31) == 0) mbar_arrive(empty, kUnitsPerWarp);
    if (++s == kStages) {
      s = 0;
      parity ^= 1u;
    }
  }
  if (nfacc.x != nfacc.x || nfacc.y != nfacc.y) atomicOr(a.status, 4u);
}

}  // namespace
