// adamw4.cu -- fused 4-bit AdamW optimizer step (ZIP-SR / ZE-EDEN) for B200
// (sm_100a), and the C ABI declared in include/adamw4.h.
//
// One kernel launch per step covers every parameter tensor.  The work is a flat
// list of 128-value units: each block of a 4-bit tensor is one unit, and each
// fp32-state tensor is cut into 128-element chunks.  The grid is persistent
// (SM count x resident CTAs) and the units are dealt out round-robin, so all
// SMs stream one contiguous window of HBM.
//
// A CTA has one producer warp and eight consumer warps.  Each consumer
// half-warp owns a ring of kStages shared-memory stages; producer lane j feeds
// the ring of half-warp j.  For every unit the producer writes a 64-byte header
// (addresses, block index, tensor id, flags, decay) into the stage and, for a
// whole 4-bit block, fills the stage with TMA bulk copies (cp.async.bulk: 512 B
// of fp32 weights, 256 B of bf16 grads, 64 + 64 B of codes) plus two 4-byte
// cp.async copies of the block scales, all completing on the stage's "full"
// mbarrier.  The consumer half-warp waits on it, computes from the stage,
// stores the results straight to global memory and hands the stage back on
// its "empty" mbarrier.  Units that are not whole
// 4-bit blocks (a ragged last block, fp32-state chunks) carry only the header
// and are read from global memory by the consumer.  Every wait is bounded by
// a timer; on expiry the kernel records the failure in a status word and the
// waiting warp leaves.
//
// Per unit, following the method flowchart of "ZIP-SR / ZE-EDEN: 4-bit AdamW
// state quantization" (daiwk.github.io, Method): decode the prior moments,
// update them, update the weights, requantise (ZIP-SR or ZE-EDEN for v, NF4 for
// m), pack.  The weights use the unquantised working moments (same page, Core
// equation: weights are updated before the moments are quantised).
//
// Arithmetic follows one fixed binary32 evaluation order with IEEE division
// and square root (__fdiv_rn, __fsqrt_rn) and fused multiply-add only where
// written (__fmaf_rn, or __ffma2_rn on value pairs, which rounds each lane like
// __fmaf_rn); the file is built with -fmad=false so nothing else is contracted.
// With that, codes, scales and weights are reproducible bit for bit by any
// IEEE implementation of the same order.
//
// No tensor cores: the step is a streaming codec, bound by HBM bandwidth.  No
// TMA multicast: every copy is this GPU's global memory into its own CTA.

#include <cuda_runtime.h>

#include <algorithm>
#include <cfloat>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <set>
#include <string>
#include <vector>

#include "../../include/adamw4.h"
#include "nf4_table.h"

namespace {

constexpr int kBlock = ADAMW4_BLOCK;              // values per quantisation block
constexpr int kLanesPerUnit = 16;                 // a half-warp per block
constexpr int kPerLane = kBlock / kLanesPerUnit;  // 8 values per lane
constexpr int kConsumerThreads = 256;             // eight consumer warps
constexpr int kCtaThreads = kConsumerThreads + 32;  // plus the producer warp
constexpr int kHalves = kConsumerThreads / kLanesPerUnit;  // consumer half-warps per CTA
constexpr int kProducerWarp = kConsumerThreads / 32;
constexpr int kStages = 3;                        // tiles in flight per CTA
// A tile is kHalves consecutive units; stage layout (CTA-wide):
//   16 unit headers (64 B each) | w 16 x 512 B | g 16 x 256 B |
//   m codes 16 x 64 B | v codes 16 x 64 B | m scales 16 x 4 B | v scales 16 x 4 B
constexpr int kOffHdr = 0;
constexpr int kOffW = kOffHdr + kHalves * 64;
constexpr int kOffG = kOffW + kHalves * 512;
constexpr int kOffMC = kOffG + kHalves * 256;
constexpr int kOffVC = kOffMC + kHalves * 64;
constexpr int kOffMS = kOffVC + kHalves * 64;
constexpr int kOffVS = kOffMS + kHalves * 4;
constexpr int kStageBytes = kOffVS + kHalves * 4; // 15,488 B, a 16-byte multiple
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
  uint32_t rk0[10], rk1[10];  // Philox round keys of the seed
  uint32_t r0_hi_k0, r0_lo;   // round 0 with counter word 2 = t: hi(M1 t) ^ key0, lo(M1 t)
  int lm_sr_active;      // final-10% LM-head phase
  uint32_t* status;      // device status word (bit 0: a pipeline wait timed out)
  int fault_stall;       // test hook: mark stages filled without filling them
};

// Code tables, passed by value and staged in shared memory by each CTA.
struct CodeTables {
  float nf4[16];        // NF4 levels, ascending
  float nf4_gap[16];    // nf4[j+1] - nf4[j]
  float vz[16];         // ZIP-SR code points k/15
  float vz_sqrt[16];    // sqrt(k/15)
  float vz_mid[16];     // nearest-point thresholds of the k/15 code (15 used)
  float2 rtn[128];      // NF4 nearest-level buckets: .x threshold, .y base code (int bits)
};

struct StateArena {
  uint8_t* mcodes;   // 64 bytes per block, element 2i in the low nibble of byte i
  uint8_t* vcodes;
  float* mscale;     // one per block
  float* vscale;
  float* fm;         // fp32-state tensors
  float* fv;
};

// What the producer tells the consumer about one unit (64 bytes).
struct __align__(16) UnitHeader {
  float* w;              // the unit's first weight
  const uint16_t* g;     // its first gradient
  uint64_t e0;           // index of that element within its (logical) tensor
  uint64_t state;        // 4-bit: block index in the code arena; fp32: element index
  uint32_t tensor_id;
  uint32_t flags;        // ADAMW4_T_* | kKindFp32 | kStaged
  float decay;           // 1 - lr * weight_decay of the tensor
  int32_t nvalid;        // values in the unit (1..128)
  uint32_t w_soff;       // bf16-weight units: stage offset of the unit's weights
  uint32_t pad_[3];
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

__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
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

// The producer's wait for a stage to come back: the consumers take
// microseconds per tile, so it naps between polls instead of taking issue
// slots from them.  False if `limit_ns` passed first.
__device__ __forceinline__ bool wait_phase_napping(uint32_t bar, uint32_t parity,
                                                   uint64_t limit_ns) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    __nanosleep(1000);
    if (mbar_test_wait(bar, parity)) return true;
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
__device__ __forceinline__ uint4 philox4x32_10(uint64_t quad, uint32_t c3, const StepArgs& a) {
  const uint64_t q0 = (uint64_t)kPhiloxM0 * (uint32_t)quad;
  uint4 c = make_uint4(a.r0_hi_k0 ^ (uint32_t)(quad >> 32), a.r0_lo,
                       (uint32_t)(q0 >> 32) ^ c3 ^ a.rk1[0], (uint32_t)q0);
#pragma unroll
  for (int r = 1; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)kPhiloxM0 * c.x;
    const uint64_t p1 = (uint64_t)kPhiloxM1 * c.z;
    c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ a.rk0[r], (uint32_t)p1,
                   (uint32_t)(p0 >> 32) ^ c.w ^ a.rk1[r], (uint32_t)p0);
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

// The eight draw words of one lane: elements 4*quad .. 4*quad + 7.
__device__ __forceinline__ void words8(const StepArgs& a, uint32_t tensor_id, uint32_t stream,
                                       uint64_t quad, uint32_t r[8]) {
  const uint32_t c3 = tensor_id * 2u + stream;
  const uint4 r0 = philox4x32_10(quad, c3, a);
  const uint4 r1 = philox4x32_10(quad + 1, c3, a);
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

// Max of non-negative binary32 values over a half-warp: their bit patterns
// order like the values, so an integer reduction gives the exact maximum.
__device__ __forceinline__ float hmax16_nonneg(float v, unsigned mask) {
  return __uint_as_float(__reduce_max_sync(mask, __float_as_uint(v)));
}

// Balanced pairwise sum of (x, y) pairs over the half-warp: partner offsets 1,
// 2, 4, 8 join adjacent 8-value groups in index order (IEEE addition is
// commutative, so both partners hold the same bits).
__device__ __forceinline__ float2 hsum16_tree2(float2 v, unsigned mask) {
#pragma unroll
  for (int off = 1; off < 16; off <<= 1) {
    const float2 o = make_float2(__shfl_xor_sync(mask, v.x, off), __shfl_xor_sync(mask, v.y, off));
    v = __fadd2_rn(v, o);
  }
  return v;
}

// NF4 nearest level: #{j : x > mid[j]}.  Bucket round(32 x + 32) holds at most
// one threshold; the table has 128 entries so any 7-bit index stays inside.
__device__ __forceinline__ uint32_t nf4_rtn_bucket(float x, float bucket_sum, const float2* rtn) {
  const float2 e = rtn[__float_as_uint(bucket_sum) & 127u];
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
  float2 rtn[128];
  float nf4[16];
  float gap[16];
  float vz[16];        // ZIP-SR code points k/15
  float4 zip[16];      // for k0 = nearest integer to 15x: {VZ[k0] (+inf for 15),
                       //   sqrt VZ[k0-1], sqrt VZ[k0], sqrt VZ[k0+1]}
  float2 vzp[16];      // {k/15, (k+1)/15}
  float vzmid[16];     // thresholds between adjacent k/15 code points
};

// ---------------------------------------------------------------------------
// Requantisation of one 4-bit block held by a half-warp (8 values per lane).
// FULL: all 128 values valid.  Otherwise `myn` values of this lane are valid.
// ---------------------------------------------------------------------------

// ZIP-SR codes of 8 values.  FLAT: also test for d(a) == d(b), which needs the
// state-space fallback; callers skip it when the block's R makes that
// impossible.
template <bool FULL, bool FLAT>
__device__ __forceinline__ uint32_t zipsr_codes8(const StepArgs& a, const SmemTables& S,
                                                 const float (&v1)[kPerLane],
                                                 const float (&den)[kPerLane],
                                                 const uint32_t (&rw)[kPerLane], float inv,
                                                 float R, int myn) {
  // two values at a time; from the last pair to the first, so that element i
  // ends in bits 4i..4i+3
  uint32_t vco = 0;
#pragma unroll
  for (int j = kPerLane / 2 - 1; j >= 0; --j) {
    const float2 x2 = __fmul2_rn(make_float2(v1[2 * j], v1[2 * j + 1]), f2(inv));
    const float2 t2 = __ffma2_rn(x2, f2(15.0f), f2(kMagic));
    // k0, the nearest integer to 15x, is the bracket or one above it (the top
    // entry's threshold is +inf: its bracket is always 14)
    const uint32_t k0a = __float_as_uint(t2.x) & 15u, k0b = __float_as_uint(t2.y) & 15u;
    const float4 ea = S.zip[k0a], eb = S.zip[k0b];
    const bool deca = x2.x < ea.x, decb = x2.y < eb.x;
    // square roots of the lower and upper code points of each value
    const float2 sa = make_float2(deca ? ea.y : ea.z, decb ? eb.y : eb.z);
    const float2 sb = make_float2(deca ? ea.z : ea.w, decb ? eb.z : eb.w);
    const float2 da = __ffma2_rn(sa, f2(R), f2(a.eps));
    const float2 db = __ffma2_rn(sb, f2(R), f2(a.eps));
    const float2 dv = make_float2(den[2 * j], den[2 * j + 1]);
    // fma(y, -1, x) rounds like x - y
    const float2 B = __fmul2_rn(__ffma2_rn(da, f2(-1.0f), db), dv);      // (db - da) * dv
    const float2 rhs = __fmul2_rn(__ffma2_rn(dv, f2(-1.0f), db), da);    // (db - dv) * da
    const float2 f = make_float2(one_plus_u(rw[2 * j]), one_plus_u(rw[2 * j + 1]));
    const float2 lhs = __ffma2_rn(f, B, make_float2(-B.x, -B.y));         // u * B
    bool lowa = lhs.x < rhs.x, lowb = lhs.y < rhs.y;
    const uint32_t ka = k0a - (deca ? 1u : 0u), kb = k0b - (decb ? 1u : 0u);
    if (FLAT) {
      if (da.x == db.x) {
        const float2 z = S.vzp[ka];
        lowa = __fmul_rn(__fsub_rn(f.x, 1.0f), __fsub_rn(z.y, z.x)) < __fsub_rn(z.y, x2.x);
      }
      if (da.y == db.y) {
        const float2 z = S.vzp[kb];
        lowb = __fmul_rn(__fsub_rn(f.y, 1.0f), __fsub_rn(z.y, z.x)) < __fsub_rn(z.y, x2.y);
      }
    }
    const uint32_t ca = (FULL || 2 * j < myn) ? ka + (lowa ? 0u : 1u) : 0u;
    const uint32_t cb = (FULL || 2 * j + 1 < myn) ? kb + (lowb ? 0u : 1u) : 0u;
    vco = (vco * 16u + cb) * 16u + ca;
  }
  return vco;
}

template <int VCODE, bool FULL>
__device__ __forceinline__ void requant_store(const StepArgs& a, const SmemTables& S,
                                              uint32_t tensor_id, uint32_t flags, uint64_t e0,
                                              int lane, int myn, unsigned hmask,
                                              const float (&m1)[kPerLane],
                                              const float (&v1)[kPerLane],
                                              const float (&den)[kPerLane], uint32_t* mcw,
                                              uint32_t* vcw, float* msp, float* vsp) {
  float am = 0.0f, av = 0.0f;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    if (FULL || i < myn) {
      am = fmaxf(am, fabsf(m1[i]));
      av = fmaxf(av, fabsf(v1[i]));
    }
  }
  am = hmax16_nonneg(am, hmask);
  av = hmax16_nonneg(av, hmask);

  // ---- first moment: absmax scale, NF4 codes ----
  uint32_t mco = 0;
  float mso = 0.0f;
  if (am >= FLT_MIN) {
    const float inv = __fdiv_rn(1.0f, am);
    if ((flags & ADAMW4_T_LM_HEAD) && a.lm_sr_active) {
      uint32_t rw[kPerLane];
      words8(a, tensor_id, kStreamM, (e0 + (uint64_t)(lane * kPerLane)) >> 2, rw);
#pragma unroll
      for (int i = 0; i < kPerLane; ++i)
        if (FULL || i < myn)
          mco |= nf4_sr(__fmul_rn(m1[i], inv), uniform23(rw[i]), S.nf4, S.gap) << (4 * i);
    } else {
#pragma unroll
      for (int j = kPerLane / 2 - 1; j >= 0; --j) {   // last element first
        const float2 x = __fmul2_rn(make_float2(m1[2 * j], m1[2 * j + 1]), f2(inv));
        const float2 b = __ffma2_rn(x, f2(32.0f), f2(kMagic + 32.0f));
        const uint32_t c1 = (FULL || 2 * j + 1 < myn) ? nf4_rtn_bucket(x.y, b.y, S.rtn) : 0u;
        const uint32_t c0 = (FULL || 2 * j < myn) ? nf4_rtn_bucket(x.x, b.x, S.rtn) : 0u;
        mco = (mco * 16u + c1) * 16u + c0;
      }
    }
    mso = am;
  }

  // ---- second moment ----
  uint32_t vco = 0;
  float vso = 0.0f;
  if (av >= FLT_MIN) {
    const float inv = __fdiv_rn(1.0f, av);
    if (VCODE == kVZip) {
      // ZIP-SR ("ZIP-SR / ZE-EDEN", Core equation): keep the lower code point
      // with probability [h(v)-h(b)]/[h(a)-h(b)], evaluated division-free as
      // u*((db-da)*dv) < (db-dv)*da with d = 1/h.
      const float R = __fmul_rn(__fsqrt_rn(av), a.rs_bc2);
      uint32_t rw[kPerLane];
      words8(a, tensor_id, kStreamV, (e0 + (uint64_t)(lane * kPerLane)) >> 2, rw);
      // d(a) == d(b) needs (sqrt(k+1/15) - sqrt(k/15)) R below two ulps of
      // R + eps; the smallest gap is 0.0339, so R > 1e-5 eps rules it out.
      if (R > __fmul_rn(1e-5f, a.eps) && a.eps >= FLT_MIN)
        vco = zipsr_codes8<FULL, false>(a, S, v1, den, rw, inv, R, myn);
      else
        vco = zipsr_codes8<FULL, true>(a, S, v1, den, rw, inv, R, myn);
      vso = av;
    } else if (VCODE == kVZiRtn || VCODE == kVZiSr) {
      // State-space rules on the zero-inclusive code: nearest code point, or
      // the lower one with probability (b - x)/(b - a).
      uint32_t rw[kPerLane];
      if (VCODE == kVZiSr) words8(a, tensor_id, kStreamV, (e0 + (uint64_t)(lane * kPerLane)) >> 2, rw);
#pragma unroll
      for (int j = kPerLane / 2 - 1; j >= 0; --j) {   // last element first
        const float2 x2 = __fmul2_rn(make_float2(v1[2 * j], v1[2 * j + 1]), f2(inv));
        const float2 t2 = __ffma2_rn(x2, f2(15.0f), f2(kMagic));
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
            const bool lower = __fmul_rn(uniform23(rw[i]), __fsub_rn(z.y, z.x)) < __fsub_rn(z.y, x);
            c = k + (lower ? 0u : 1u);
          }
          vco = vco * 16u + ((FULL || i < myn) ? c : 0u);
        }
      }
      vso = av;
    } else if (VCODE == kVZeFloor) {
      // Zero-excluded code with a positive floor: nearest (k+1)/16, no rescale.
#pragma unroll
      for (int j = kPerLane / 2 - 1; j >= 0; --j) {
        const float2 x2 = __fmul2_rn(make_float2(v1[2 * j], v1[2 * j + 1]), f2(inv));
        const float2 t2 = __ffma2_rn(x2, f2(16.0f), f2(kMagic));   // kMagic + rint(16x)
        const uint32_t k0 = max(__float_as_uint(t2.x) & 31u, 1u) - 1u;
        const uint32_t k1 = max(__float_as_uint(t2.y) & 31u, 1u) - 1u;
        const uint32_t c1 = (FULL || 2 * j + 1 < myn) ? k1 : 0u;
        const uint32_t c0 = (FULL || 2 * j < myn) ? k0 : 0u;
        vco = (vco * 16u + c1) * 16u + c0;
      }
      vso = av;
    } else {
      // ZE-EDEN ("ZIP-SR / ZE-EDEN", Core equation): nearest zero-excluded
      // code point, scale times ||x||^2 / max(<x,Q(x)>, 1e-12 s^2) on x = v/s.
      float2 l1[kPerLane / 2];
#pragma unroll
      for (int j = 0; j < kPerLane / 2; ++j) {
        const float2 x2 = __fmul2_rn(make_float2(v1[2 * j], v1[2 * j + 1]), f2(inv));
        const float2 t2 = __ffma2_rn(x2, f2(16.0f), f2(kMagic));   // kMagic + rint(16x)
        const float2 c2 = __fadd2_rn(t2, f2(-kMagic));             // rint(16x), exact
        const float2 q2 = __fmul2_rn(make_float2(fmaxf(c2.x, 1.0f), fmaxf(c2.y, 1.0f)),
                                     f2(0.0625f));                 // (k+1)/16
        const uint32_t k0 = max(__float_as_uint(t2.x) & 31u, 1u) - 1u;
        const uint32_t k1 = max(__float_as_uint(t2.y) & 31u, 1u) - 1u;
        float2 xx = __fmul2_rn(x2, x2);
        float2 xq = __fmul2_rn(x2, q2);
        if (!FULL) {
          if (2 * j >= myn) { xx.x = 0.0f; xq.x = 0.0f; }
          if (2 * j + 1 >= myn) { xx.y = 0.0f; xq.y = 0.0f; }
        }
        if (FULL || 2 * j < myn) vco |= k0 << (8 * j);
        if (FULL || 2 * j + 1 < myn) vco |= k1 << (8 * j + 4);
        // first tree level: (x0^2 + x1^2, x0 q0 + x1 q1)
        l1[j] = __fadd2_rn(make_float2(xx.x, xq.x), make_float2(xx.y, xq.y));
      }
      const float2 l2a = __fadd2_rn(l1[0], l1[1]);
      const float2 l2b = __fadd2_rn(l1[2], l1[3]);
      const float2 s = hsum16_tree2(__fadd2_rn(l2a, l2b), hmask);    // (sum x^2, sum x q)
      vso = __fmul_rn(av, __fdiv_rn(s.x, fmaxf(s.y, 1e-12f)));
    }
  }

  *mcw = mco;
  *vcw = vco;
  if (lane == 0) {
    *msp = mso;
    *vsp = vso;
  }
}

// Decode + moment update + weight update for 8 values of a 4-bit block.
__device__ __forceinline__ void update8(const StepArgs& a, const SmemTables& S, float decay,
                                        float (&w)[kPerLane], const float (&g)[kPerLane],
                                        uint32_t mc, uint32_t vc, float sm, float sv,
                                        float (&m1)[kPerLane], float (&v1)[kPerLane],
                                        float (&den)[kPerLane]) {
#pragma unroll
  for (int j = 0; j < kPerLane / 2; ++j) {
    // one byte holds the codes of values 2j (low nibble) and 2j+1 (high nibble)
    const float2 m0 = __fmul2_rn(S.mpair[__byte_perm(mc, 0, 0x4440 + j)], f2(sm));
    const float2 v0 = __fmul2_rn(S.vpair[__byte_perm(vc, 0, 0x4440 + j)], f2(sv));
    const float2 gg = make_float2(g[2 * j], g[2 * j + 1]);
    const float2 mm = __ffma2_rn(f2(a.b1), m0, __fmul2_rn(f2(a.omb1), gg));
    const float2 vv = __ffma2_rn(f2(a.b2), v0, __fmul2_rn(f2(a.omb2), __fmul2_rn(gg, gg)));
    const float2 dd = __ffma2_rn(make_float2(__fsqrt_rn(vv.x), __fsqrt_rn(vv.y)), f2(a.rs_bc2),
                                 f2(a.eps));
    const float2 qq = make_float2(__fdiv_rn(mm.x, dd.x), __fdiv_rn(mm.y, dd.y));
    const float2 ww = __ffma2_rn(f2(-a.step_size), qq,
                                 __fmul2_rn(make_float2(w[2 * j], w[2 * j + 1]), f2(decay)));
    w[2 * j] = ww.x; w[2 * j + 1] = ww.y;
    m1[2 * j] = mm.x; m1[2 * j + 1] = mm.y;
    v1[2 * j] = vv.x; v1[2 * j + 1] = vv.y;
    den[2 * j] = dd.x; den[2 * j + 1] = dd.y;
  }
}

// Weight i of a lane's run, fp32 or (BF16W and flagged) bf16.
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
// chunk of an fp32-state tensor.
template <int VCODE, bool BF16W>
__device__ __forceinline__ void process_direct(const StepArgs& a, const SmemTables& S,
                                            const StateArena& st, const UnitHeader* hdp,
                                            int lane, unsigned hmask) {
  const int my0 = lane * kPerLane;
  const int myn = min(max(hdp->nvalid - my0, 0), kPerLane);
  const uint32_t flags = hdp->flags;
  const bool wbf = BF16W && (flags & kBf16W);
  const float decay = hdp->decay;
  const uint64_t state = hdp->state;
  // the header's w is the unit's first weight, of either width
  float* wp = wbf ? nullptr : hdp->w + my0;
  uint16_t* wp16 = wbf ? reinterpret_cast<uint16_t*>(hdp->w) + my0 : nullptr;
  const uint16_t* gp = hdp->g + my0;
  float w[kPerLane], g[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    w[i] = (i < myn) ? load_w<BF16W>(wp, wp16, wbf, i) : 0.0f;
    g[i] = (i < myn) ? __uint_as_float((uint32_t)gp[i] << 16) : 0.0f;
  }
  if (flags & kKindFp32) {
    float* mp = st.fm + state + my0;
    float* vp = st.fv + state + my0;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      if (i < myn) {
        const float m1 = __fmaf_rn(a.b1, mp[i], __fmul_rn(a.omb1, g[i]));
        const float v1 = __fmaf_rn(a.b2, vp[i], __fmul_rn(a.omb2, __fmul_rn(g[i], g[i])));
        const float den = __fmaf_rn(__fsqrt_rn(v1), a.rs_bc2, a.eps);
        store_w<BF16W>(wp, wp16, wbf, i,
                       __fmaf_rn(-a.step_size, __fdiv_rn(m1, den), __fmul_rn(w[i], decay)));
        mp[i] = m1;
        vp[i] = v1;
      }
    }
    return;
  }
  const uint64_t blk = state;
  uint32_t* mcw = reinterpret_cast<uint32_t*>(st.mcodes + blk * (kBlock / 2)) + lane;
  uint32_t* vcw = reinterpret_cast<uint32_t*>(st.vcodes + blk * (kBlock / 2)) + lane;
  float m1[kPerLane], v1[kPerLane], den[kPerLane];
  update8(a, S, decay, w, g, *mcw, *vcw, st.mscale[blk], st.vscale[blk], m1, v1, den);
#pragma unroll
  for (int i = 0; i < kPerLane; ++i)
    if (i < myn) store_w<BF16W>(wp, wp16, wbf, i, w[i]);
  requant_store<VCODE, false>(a, S, hdp->tensor_id, flags, hdp->e0, lane, myn, hmask, m1, v1,
                              den, mcw, vcw, st.mscale + blk, st.vscale + blk);
}

// ---------------------------------------------------------------------------
// Producer: fills CTA-wide stages, one tile of kHalves consecutive units each.
// Lane i handles unit i of the tile (header, scales); the lane that starts a
// run of whole 4-bit blocks of one tensor issues that run's bulk copies.
// ---------------------------------------------------------------------------
template <bool BF16W>
__device__ __forceinline__ void produce(const DevTensor* __restrict__ T, int64_t u_begin,
                                        int64_t u_end, const StepArgs& a, const StateArena& st,
                                        uint8_t* stages, uint32_t full0, uint32_t empty0,
                                        int lane) {
  constexpr unsigned kMask = (1u << kHalves) - 1u;
  const int64_t ntiles = (u_end - u_begin + kHalves - 1) / kHalves;
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
    if (round > 0 && !__all_sync(kMask, wait_phase_napping(empty0 + 8u * s, (round - 1) & 1u,
                                                           kWaitLimitNs))) {
      // Leaving early: flag it, then wait (bounded) for the copies this warp
      // issued into stages not yet handed back.  Stage j was last filled in
      // this round if j < s, else in the previous one; its full barrier
      // completes that fill's phase once the bytes have landed.
      if (lane == 0) atomicOr(a.status, 1u);
      for (int j = 0; j < kStages; ++j) {
        const uint32_t last = (j < s) ? round : round - 1;
        wait_phase_napping(full0 + 8u * j, last & 1u, kDrainLimitNs);
      }
      cp_async_wait_all();
      return;
    }
    const int64_t u = u_begin + tile * kHalves + lane;
    const bool has = u < u_end;
    if (has && u >= t_end) {
      do {
        ++ti;
        t_end = __ldg(&T[ti].unit_end);
      } while (u >= t_end);
      const DevTensor* d = &T[ti];
      t_begin = __ldg(&d->unit_begin);
      t_numel = __ldg(&d->numel);
      t_soff = __ldg(&d->state_off);
      t_eoff = (int64_t)__ldg(&d->block_offset) * kBlock;
      t_param = d->param;
      t_grad = d->grad;
      t_id = __ldg(&d->tensor_id);
      t_flags = __ldg(&d->flags);
      t_decay = (float)(1.0 - (double)a.lr * (double)__ldg(&d->weight_decay));
    }
    const int64_t ub = u - t_begin;
    const int64_t e0 = ub * kBlock;
    const int nvalid = has ? (int)min((int64_t)kBlock, t_numel - e0) : 0;
    const bool staged = has && !(t_flags & kKindFp32) && nvalid == kBlock;
    const bool wbf = BF16W && (t_flags & kBf16W);       // bf16 weights: 256 B per unit
    uint8_t* sp = stages + s * kStageBytes;
    UnitHeader* hd = reinterpret_cast<UnitHeader*>(sp + kOffHdr) + lane;
    hd->w = wbf ? reinterpret_cast<float*>(reinterpret_cast<uint16_t*>(t_param) + e0)
                : t_param + e0;
    hd->g = t_grad + e0;
    hd->e0 = (uint64_t)(t_eoff + e0);   // keys the draws
    hd->state = (t_flags & kKindFp32) ? (uint64_t)(t_soff + e0) : (uint64_t)(t_soff + ub);
    hd->tensor_id = t_id;
    hd->flags = has ? (t_flags | (staged ? kStaged : 0u)) : kNoUnit;
    hd->decay = t_decay;
    hd->nvalid = nvalid;
    // Runs of whole blocks of one tensor are contiguous in global memory and
    // in the stage: one bulk copy per array per run.
    const unsigned staged_mask = __ballot_sync(kMask, staged);
    const int prev_ti = __shfl_up_sync(kMask, ti, 1);
    const bool cont = staged && lane > 0 && ((staged_mask >> (lane - 1)) & 1u) && prev_ti == ti;
    const unsigned cont_mask = __ballot_sync(kMask, cont);
    const uint32_t dst = stages_s + (uint32_t)(s * kStageBytes);
    uint32_t tx = (uint32_t)__popc(staged_mask) * kUnitTx;
    if (BF16W) tx -= (uint32_t)__popc(__ballot_sync(kMask, staged && wbf)) * 256u;
    if (lane == 0) mbar_arrive_expect_tx(full, tx);
    if (BF16W) {
      // A run's weights land packed at the start of its own units' 512-B w
      // slots: 512 B per unit for fp32, 256 B for bf16.  The run starts at the
      // nearest lane at or below this one that does not continue a run.
      const int start = 31 - __clz(~cont_mask & ((2u << lane) - 1u));
      hd->w_soff = (uint32_t)(kOffW + start * 512 + (lane - start) * (wbf ? 256 : 512));
    }
    if (staged && !cont && !a.fault_stall) {
      // this lane starts a run: it extends over the following lanes whose
      // unit continues it
      const unsigned rest = ~(cont_mask >> (lane + 1));
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
      cp_async4(dst + kOffMS + lane * 4, st.mscale + blk);
      cp_async4(dst + kOffVS + lane * 4, st.vscale + blk);
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

// ---------------------------------------------------------------------------
// The step kernel
// ---------------------------------------------------------------------------

template <int VCODE, bool BF16W>
__global__ void __launch_bounds__(kCtaThreads, 3)
adamw4_step_kernel(const DevTensor* __restrict__ T, int64_t u_begin, int64_t u_end, StepArgs a,
                   CodeTables tabs, StateArena st) {
  extern __shared__ __align__(128) uint8_t s_stage[];
  __shared__ __align__(8) uint64_t s_full[kStages];
  __shared__ __align__(8) uint64_t s_empty[kStages];
  __shared__ SmemTables S;

  {
    const int t = threadIdx.x;
    if (t < 256) {
      S.mpair[t] = make_float2(tabs.nf4[t & 15], tabs.nf4[t >> 4]);
      const bool zx = (VCODE == kVZe || VCODE == kVZeFloor);   // zero-excluded code
      const float lo = zx ? __fmul_rn((float)((t & 15) + 1), 0.0625f) : tabs.vz[t & 15];
      const float hi = zx ? __fmul_rn((float)((t >> 4) + 1), 0.0625f) : tabs.vz[t >> 4];
      S.vpair[t] = make_float2(lo, hi);
    }
    if (t < 128) S.rtn[t] = tabs.rtn[t];
    if (t < 16) {
      S.nf4[t] = tabs.nf4[t];
      S.gap[t] = tabs.nf4_gap[t];
      S.vz[t] = tabs.vz[t];
      S.zip[t] = make_float4(t == 15 ? INFINITY : tabs.vz[t], tabs.vz_sqrt[max(t - 1, 0)],
                             tabs.vz_sqrt[t], tabs.vz_sqrt[min(t + 1, 15)]);
      S.vzp[t] = make_float2(tabs.vz[t], tabs.vz[min(t + 1, 15)]);
      S.vzmid[t] = tabs.vz_mid[t];
    }
    if (t < kStages) {
      // full: the producer's expect-tx arrive plus one cp.async arrive per
      // producer lane; empty: one release per consumer half-warp
      mbar_init(smem_addr(&s_full[t]), 1 + kHalves);
      mbar_init(smem_addr(&s_empty[t]), kHalves);
    }
    fence_mbar_init();
  }
  __syncthreads();

  const uint32_t full0 = smem_addr(&s_full[0]);
  const uint32_t empty0 = smem_addr(&s_empty[0]);
  const int warp = threadIdx.x >> 5;
  if (warp == kProducerWarp) {
    const int lane = threadIdx.x & 31;
    if (lane < kHalves) produce<BF16W>(T, u_begin, u_end, a, st, s_stage, full0, empty0, lane);
    return;
  }

  // ---- consumers: half-warp `half` takes unit `half` of every tile ----
  const int lane = threadIdx.x & 15;
  const int half = threadIdx.x >> 4;
  const unsigned hmask = 0xFFFFu << (threadIdx.x & 16);
  const int64_t ntiles = (u_end - u_begin + kHalves - 1) / kHalves;
  int s = 0;
  uint32_t parity = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const uint32_t full = full0 + 8u * s;
    const uint32_t empty = empty0 + 8u * s;
    if (!__all_sync(hmask, wait_phase(full, parity, kWaitLimitNs))) {
      if (lane == 0) atomicOr(a.status, 1u);
      return;
    }
    const uint8_t* sp = s_stage + s * kStageBytes;
    const UnitHeader* hdp = reinterpret_cast<const UnitHeader*>(sp + kOffHdr) + half;
    const uint32_t flags = hdp->flags;
    if (flags & kStaged) {
      float w[kPerLane], g[kPerLane];
      const bool wbf = BF16W && (flags & kBf16W);
      {
        const uint4 gg = *reinterpret_cast<const uint4*>(sp + kOffG + half * 256 + lane * 16);
        if (wbf) {
          const uint4 wr = *reinterpret_cast<const uint4*>(sp + hdp->w_soff + lane * 16);
          w[0] = bf16lo(wr.x); w[1] = bf16hi(wr.x); w[2] = bf16lo(wr.y); w[3] = bf16hi(wr.y);
          w[4] = bf16lo(wr.z); w[5] = bf16hi(wr.z); w[6] = bf16lo(wr.w); w[7] = bf16hi(wr.w);
        } else {
          const uint8_t* wsrc = sp + kOffW + half * 512 + lane * 32;
          const float4 wa = *reinterpret_cast<const float4*>(wsrc);
          const float4 wb = *reinterpret_cast<const float4*>(wsrc + 16);
          w[0] = wa.x; w[1] = wa.y; w[2] = wa.z; w[3] = wa.w;
          w[4] = wb.x; w[5] = wb.y; w[6] = wb.z; w[7] = wb.w;
        }
        g[0] = bf16lo(gg.x); g[1] = bf16hi(gg.x); g[2] = bf16lo(gg.y); g[3] = bf16hi(gg.y);
        g[4] = bf16lo(gg.z); g[5] = bf16hi(gg.z); g[6] = bf16lo(gg.w); g[7] = bf16hi(gg.w);
      }
      const uint32_t mc = *reinterpret_cast<const uint32_t*>(sp + kOffMC + half * 64 + lane * 4);
      const uint32_t vc = *reinterpret_cast<const uint32_t*>(sp + kOffVC + half * 64 + lane * 4);
      const float sm = *reinterpret_cast<const float*>(sp + kOffMS + half * 4);
      const float sv = *reinterpret_cast<const float*>(sp + kOffVS + half * 4);

      float m1[kPerLane], v1[kPerLane], den[kPerLane];
      update8(a, S, hdp->decay, w, g, mc, vc, sm, sv, m1, v1, den);
      if (wbf) {
        uint16_t* wp = reinterpret_cast<uint16_t*>(hdp->w) + lane * kPerLane;
        *reinterpret_cast<uint4*>(wp) = make_uint4(bf16x2_rn(w[0], w[1]), bf16x2_rn(w[2], w[3]),
                                                   bf16x2_rn(w[4], w[5]), bf16x2_rn(w[6], w[7]));
      } else {
        float* wp = hdp->w + lane * kPerLane;
        *reinterpret_cast<float4*>(wp) = make_float4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<float4*>(wp + 4) = make_float4(w[4], w[5], w[6], w[7]);
      }
      const uint64_t blk = hdp->state;
      uint32_t* mcw = reinterpret_cast<uint32_t*>(st.mcodes + blk * (kBlock / 2)) + lane;
      uint32_t* vcw = reinterpret_cast<uint32_t*>(st.vcodes + blk * (kBlock / 2)) + lane;
      requant_store<VCODE, true>(a, S, hdp->tensor_id, flags, hdp->e0, lane, kPerLane, hmask, m1,
                                 v1, den, mcw, vcw, st.mscale + blk, st.vscale + blk);
    } else if (!(flags & kNoUnit)) {
      process_direct<VCODE, BF16W>(a, S, st, hdp, lane, hmask);
    }
    // every read of the stage (header included) is done: hand it back
    fence_proxy_async_smem();
    __syncwarp(hmask);
    if (lane == 0) mbar_arrive(empty, 1);
    if (++s == kStages) {
      s = 0;
      parity ^= 1u;
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

struct HostTensor {
  adamw4_tensor desc;
  bool fp32;
  int64_t nblocks;      // 4-bit: blocks; fp32: 128-element chunks
  int64_t state_off;    // 4-bit: first block; fp32: first element
  int64_t unit_begin;   // its first unit in the flat unit list
};

}  // namespace

struct adamw4_handle {
  int device = 0;
  adamw4_config cfg{};
  int64_t t = 0;
  std::vector<HostTensor> tensors;
  DevTensor* d_tensors = nullptr;
  void* d_arena = nullptr;
  size_t arena_bytes = 0;
  StateArena st{};
  int64_t nblocks4 = 0;       // 4-bit blocks
  int64_t nfp32 = 0;          // fp32 arena elements (with alignment)
  int64_t nunits = 0;
  bool bf16w = false;             // some tensor keeps bf16 weights
  int grid = 0;
  uint32_t* d_status = nullptr;   // device status word (in the arena)
  cudaStream_t s_in = nullptr;    // adamw4_step_host: host-to-device copies
  cudaStream_t s_out = nullptr;   // adamw4_step_host: device-to-host copies
  std::vector<cudaEvent_t> events;
  int fault_stall = 0;            // test hook for the next step
  CodeTables tabs{};
  std::string err;
};

namespace {

std::mutex g_mu;
std::set<const adamw4_handle*> g_live;
thread_local std::string t_err;

bool live(const adamw4_handle* h) {
  std::lock_guard<std::mutex> lk(g_mu);
  return h != nullptr && g_live.count(h) != 0;
}

int fail(adamw4_handle* h, int code, const std::string& msg) {
  t_err = msg;
  if (h != nullptr) h->err = msg;
  return code;
}

int cuda_fail(adamw4_handle* h, cudaError_t e, const char* what) {
  return fail(h, ADAMW4_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// Restores the caller's current device on scope exit.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  cudaError_t err = cudaSuccess;
  explicit DeviceGuard(int dev) {
    err = cudaGetDevice(&prev);
    if (err != cudaSuccess) return;
    if (prev != dev) err = cudaSetDevice(dev);
    ok = (err == cudaSuccess);
  }
  ~DeviceGuard() {
    if (ok && prev >= 0) cudaSetDevice(prev);
  }
};

void build_tables(CodeTables* T) {
  for (int j = 0; j < 16; ++j) T->nf4[j] = kNF4Levels[j];
  for (int j = 0; j < 15; ++j) T->nf4_gap[j] = kNF4Levels[j + 1] - kNF4Levels[j];
  T->nf4_gap[15] = 0.0f;
  for (int k = 0; k < 16; ++k) {
    volatile float num = (float)k;
    T->vz[k] = num / 15.0f;
    T->vz_sqrt[k] = std::sqrt(T->vz[k]);
  }
  for (int k = 0; k < 15; ++k)
    T->vz_mid[k] = (float)(((double)T->vz[k] + (double)T->vz[k + 1]) * 0.5);
  T->vz_mid[15] = INFINITY;
  // Midpoints of adjacent binary32 levels, exact in binary64, rounded once.
  float mid[15];
  for (int j = 0; j < 15; ++j)
    mid[j] = (float)(((double)kNF4Levels[j] + (double)kNF4Levels[j + 1]) * 0.5);
  // Bucket b of x is round(32 x + 32), in [0, 64] for |x| <= 1 + 2^-23 and
  // monotone in x.  A bucket holds at most one midpoint, so the nearest level
  // is the count of midpoints in lower buckets plus one comparison.
  int bucket_of[15];
  for (int j = 0; j < 15; ++j) {
    const float y = std::fma(mid[j], 32.0f, 12582944.0f);
    int32_t bits;
    std::memcpy(&bits, &y, 4);
    bucket_of[j] = std::min(std::max(bits - 0x4B400000, 0), 64);
  }
  // Indices 65..127 never occur for |x| <= 1 + 2^-23; they hold "above all".
  for (int b = 0; b < 128; ++b) {
    int base = 0;
    float thr = INFINITY;
    for (int j = 0; j < 15; ++j) {
      if (bucket_of[j] < b) ++base;
      if (bucket_of[j] == b) thr = mid[j];
    }
    int32_t base_bits = base;
    float base_f;
    std::memcpy(&base_f, &base_bits, 4);
    T->rtn[b] = make_float2(thr, base_f);
  }
}

bool tables_ok(const CodeTables& T) {
  int seen[65] = {0};
  for (int j = 0; j < 15; ++j) {
    const float mid = (float)(((double)T.nf4[j] + (double)T.nf4[j + 1]) * 0.5);
    const float y = std::fma(mid, 32.0f, 12582944.0f);
    int32_t bits;
    std::memcpy(&bits, &y, 4);
    if (++seen[std::min(std::max(bits - 0x4B400000, 0), 64)] > 1) return false;
  }
  return true;
}

// pow() in binary64 for the bias corrections; the same libm call on the host
// gives the same value wherever the scalars are formed.
StepArgs make_args(const adamw4_config& c, float lr, int64_t t) {
  StepArgs a{};
  const double bc1 = 1.0 - std::pow((double)c.beta1, (double)t);
  const double bc2 = 1.0 - std::pow((double)c.beta2, (double)t);
  a.step_size = (float)((double)lr / bc1);
  a.rs_bc2 = (float)(1.0 / std::sqrt(bc2));
  a.b1 = c.beta1;
  a.omb1 = (float)(1.0 - (double)c.beta1);
  a.b2 = c.beta2;
  a.omb2 = (float)(1.0 - (double)c.beta2);
  a.eps = c.eps;
  a.lr = lr;
  // Philox round keys: round r uses the seed words plus r times the Weyl
  // constants (mod 2^32).
  for (int r = 0; r < 10; ++r) {
    a.rk0[r] = (uint32_t)c.seed + (uint32_t)r * kPhiloxW0;
    a.rk1[r] = (uint32_t)(c.seed >> 32) + (uint32_t)r * kPhiloxW1;
  }
  const uint64_t m1t = (uint64_t)kPhiloxM1 * (uint32_t)t;
  a.r0_hi_k0 = (uint32_t)(m1t >> 32) ^ a.rk0[0];
  a.r0_lo = (uint32_t)m1t;
  a.lm_sr_active = (c.total_steps > 0) && (10 * t > 9 * c.total_steps);
  a.status = nullptr;
  a.fault_stall = 0;
  return a;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr uint32_t kUserFlags = ADAMW4_T_NORM | ADAMW4_T_LM_HEAD | ADAMW4_T_FP32_STATE |
                                ADAMW4_T_QUANT_STATE | ADAMW4_T_BF16_PARAM;

// Bytes of one weight of tensor t.
uintptr_t param_bytes(const adamw4_tensor& t) { return (t.flags & ADAMW4_T_BF16_PARAM) ? 2u : 4u; }

// fp32 state for normalisation tensors, tensors flagged FP32_STATE and tensors
// under 4096 elements -- unless QUANT_STATE marks a piece of a larger tensor
// that keeps 4-bit state.
bool fp32_state(const adamw4_tensor& t) {
  if (t.flags & (ADAMW4_T_NORM | ADAMW4_T_FP32_STATE)) return true;
  if (t.flags & ADAMW4_T_QUANT_STATE) return false;
  return t.numel < ADAMW4_MIN_QUANT_NUMEL;
}

// The flag and piece checks of one descriptor: nullptr when they pass.
const char* piece_error(const adamw4_tensor& t) {
  if (t.flags & ~kUserFlags) return "unknown flag bits";
  if ((t.flags & ADAMW4_T_QUANT_STATE) && (t.flags & (ADAMW4_T_NORM | ADAMW4_T_FP32_STATE)))
    return "QUANT_STATE cannot be combined with NORM or FP32_STATE";
  if (t.elem_offset < 0 || t.elem_offset % kBlock != 0 || t.elem_offset >= ((int64_t)1 << 39))
    return "elem_offset must be a multiple of 128 in [0, 2^39)";
  return nullptr;
}

// The kernel's descriptor of tensor x, whose units start at `unit` and whose
// state starts at `state_off`.
DevTensor dev_tensor(const adamw4_tensor& x, bool fp32, int64_t unit, int64_t state_off) {
  DevTensor d;
  d.param = x.param;
  d.grad = x.grad_bf16;
  d.numel = x.numel;
  d.unit_begin = unit;
  d.unit_end = unit + (x.numel + kBlock - 1) / kBlock;
  d.state_off = state_off;
  d.tensor_id = x.tensor_id;
  d.flags = x.flags | (fp32 ? kKindFp32 : 0u);
  d.weight_decay = x.weight_decay;
  d.block_offset = (uint32_t)(x.elem_offset / kBlock);
  return d;
}

int validate(const adamw4_config* cfg, const adamw4_tensor* ts, int n) {
  if (cfg == nullptr) return fail(nullptr, ADAMW4_EINVAL, "config is NULL");
  if (!(cfg->beta1 >= 0.0f && cfg->beta1 < 1.0f) || !(cfg->beta2 >= 0.0f && cfg->beta2 < 1.0f))
    return fail(nullptr, ADAMW4_EINVAL, "beta1 and beta2 must lie in [0, 1)");
  if (!(cfg->eps > 0.0f) || !std::isfinite(cfg->eps))
    return fail(nullptr, ADAMW4_EINVAL, "eps must be positive and finite");
  if (!(cfg->lr >= 0.0f) || !std::isfinite(cfg->lr))
    return fail(nullptr, ADAMW4_EINVAL, "lr must be finite and non-negative");
  if (cfg->vcode < ADAMW4_V_ZIPSR || cfg->vcode > ADAMW4_V_ZE_FLOOR)
    return fail(nullptr, ADAMW4_EINVAL, "vcode must be one of the adamw4_vcode values");
  if (cfg->total_steps < 0) return fail(nullptr, ADAMW4_EINVAL, "total_steps must be >= 0");
  if (n < 0 || (n > 0 && ts == nullptr))
    return fail(nullptr, ADAMW4_EINVAL, "tensor list is NULL or n < 0");
  std::set<uint32_t> ids;
  struct Range { uintptr_t lo, hi; int idx; bool param; };
  std::vector<Range> ranges;
  for (int i = 0; i < n; ++i) {
    const adamw4_tensor& t = ts[i];
    const std::string at = "tensor " + std::to_string(i) + ": ";
    if (t.param == nullptr || t.grad_bf16 == nullptr)
      return fail(nullptr, ADAMW4_EINVAL, at + "param or grad pointer is NULL");
    if (t.numel <= 0) return fail(nullptr, ADAMW4_EINVAL, at + "numel must be positive");
    if (t.numel > ((int64_t)1 << 40)) return fail(nullptr, ADAMW4_EINVAL, at + "numel too large");
    if (!aligned16(t.param) || !aligned16(t.grad_bf16))
      return fail(nullptr, ADAMW4_EALIGN, at + "param and grad must be 16-byte aligned");
    if (!std::isfinite(t.weight_decay))
      return fail(nullptr, ADAMW4_EINVAL, at + "weight_decay must be finite");
    if (const char* why = piece_error(t)) return fail(nullptr, ADAMW4_EINVAL, at + why);
    if (!ids.insert(t.tensor_id).second)
      return fail(nullptr, ADAMW4_EINVAL, at + "duplicate tensor_id " + std::to_string(t.tensor_id));
    const uintptr_t p = reinterpret_cast<uintptr_t>(t.param);
    const uintptr_t g = reinterpret_cast<uintptr_t>(t.grad_bf16);
    ranges.push_back({p, p + (uintptr_t)t.numel * param_bytes(t), i, true});
    ranges.push_back({g, g + (uintptr_t)t.numel * 2u, i, false});
  }
  // Params are written in place: no param may overlap another param or a grad.
  std::sort(ranges.begin(), ranges.end(), [](const Range& x, const Range& y) { return x.lo < y.lo; });
  uintptr_t param_hi = 0;        // highest end of a param seen so far
  uintptr_t any_hi = 0;          // highest end of any range seen so far
  int any_idx = -1, param_idx = -1;
  for (const Range& r : ranges) {
    if (r.param && r.lo < any_hi)
      return fail(nullptr, ADAMW4_EINVAL, "tensor " + std::to_string(r.idx) +
                                              ": param overlaps the buffers of tensor " +
                                              std::to_string(any_idx));
    if (!r.param && r.lo < param_hi)
      return fail(nullptr, ADAMW4_EINVAL, "tensor " + std::to_string(r.idx) +
                                              ": grad overlaps the param of tensor " +
                                              std::to_string(param_idx));
    if (r.hi > any_hi) { any_hi = r.hi; any_idx = r.idx; }
    if (r.param && r.hi > param_hi) { param_hi = r.hi; param_idx = r.idx; }
  }
  return ADAMW4_OK;
}

template <int VCODE, bool BF16W>
int occupancy_grid(int device, int* grid) {
  int sms = 0, per_sm = 0;
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) return (int)e;
  // The stage rings live in dynamic shared memory above the 48 KB default.
  e = cudaFuncSetAttribute(adamw4_step_kernel<VCODE, BF16W>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemStages);
  if (e != cudaSuccess) return (int)e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, adamw4_step_kernel<VCODE, BF16W>,
                                                    kCtaThreads, kSmemStages);
  if (e != cudaSuccess) return (int)e;
  *grid = sms * std::max(per_sm, 1);
  return 0;
}

template <bool BF16W>
int grid_for_w(int vcode, int device, int* grid) {
  switch (vcode) {
    case kVZip: return occupancy_grid<kVZip, BF16W>(device, grid);
    case kVZe: return occupancy_grid<kVZe, BF16W>(device, grid);
    case kVZiRtn: return occupancy_grid<kVZiRtn, BF16W>(device, grid);
    case kVZiSr: return occupancy_grid<kVZiSr, BF16W>(device, grid);
    case kVZeFloor: return occupancy_grid<kVZeFloor, BF16W>(device, grid);
    default: return (int)cudaErrorInvalidValue;
  }
}

// The launch grid (SM count x resident CTAs) of the instantiation for vcode,
// with (bf16w) or without support for bf16 weights.
int grid_for(int vcode, bool bf16w, int device, int* grid) {
  return bf16w ? grid_for_w<true>(vcode, device, grid) : grid_for_w<false>(vcode, device, grid);
}

template <bool BF16W>
void launch_w(int vcode, int grid, cudaStream_t s, const DevTensor* T, int64_t u0, int64_t u1,
              const StepArgs& a, const CodeTables& tabs, const StateArena& st) {
  const int n = kCtaThreads;
  const int smem = kSmemStages;
  switch (vcode) {
    case kVZip:
      adamw4_step_kernel<kVZip, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, tabs, st);
      break;
    case kVZe:
      adamw4_step_kernel<kVZe, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, tabs, st);
      break;
    case kVZiRtn:
      adamw4_step_kernel<kVZiRtn, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, tabs, st);
      break;
    case kVZiSr:
      adamw4_step_kernel<kVZiSr, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, tabs, st);
      break;
    default:
      adamw4_step_kernel<kVZeFloor, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, tabs, st);
      break;
  }
}

// Enqueues the step kernel instantiated for vcode over units [u0, u1) of the
// table; bf16w selects the instantiation that reads and writes bf16 weights
// where a tensor asks for it.
void launch_vcode(int vcode, bool bf16w, int grid, cudaStream_t s, const DevTensor* T,
                  int64_t u0, int64_t u1, const StepArgs& a, const CodeTables& tabs,
                  const StateArena& st) {
  if (bf16w) launch_w<true>(vcode, grid, s, T, u0, u1, a, tabs, st);
  else launch_w<false>(vcode, grid, s, T, u0, u1, a, tabs, st);
}

// One launch over units [u0, u1) of the handle's list.
int launch(adamw4_handle* h, StepArgs a, cudaStream_t s, int64_t u0, int64_t u1) {
  if (u1 <= u0) return ADAMW4_OK;
  const int64_t need = (u1 - u0 + kHalves - 1) / kHalves;
  const int grid = (int)std::min<int64_t>(h->grid, need);
  a.status = h->d_status;
  a.fault_stall = h->fault_stall;
  h->fault_stall = 0;
  launch_vcode(h->cfg.vcode, h->bf16w, grid, s, h->d_tensors, u0, u1, a, h->tabs, h->st);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(h, e, "step kernel launch");
  return ADAMW4_OK;
}

void release(adamw4_handle* h) {
  if (h->d_tensors) cudaFree(h->d_tensors);
  if (h->d_arena) cudaFree(h->d_arena);
  for (cudaEvent_t ev : h->events) cudaEventDestroy(ev);
  if (h->s_in) cudaStreamDestroy(h->s_in);
  if (h->s_out) cudaStreamDestroy(h->s_out);
  h->d_tensors = nullptr;
  h->d_arena = nullptr;
  h->events.clear();
  h->s_in = h->s_out = nullptr;
}

// Units per piece of the pipelined adamw4_step_host: 2^19 units (64 Mi values,
// 128 MB of grads up, 256 MB of fp32 weights down).  ADAMW4_HOST_CHUNK_UNITS
// overrides it (tests use small pieces to cut tensors at many places).
int64_t host_chunk_units() {
  if (const char* v = std::getenv("ADAMW4_HOST_CHUNK_UNITS")) {
    const long long n = std::atoll(v);
    if (n > 0) return (int64_t)n;
  }
  return (int64_t)1 << 19;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------

extern "C" int adamw4_create(const adamw4_config* cfg, const adamw4_tensor* tensors, int n,
                             int device, adamw4_handle** out) {
  if (out == nullptr) return fail(nullptr, ADAMW4_EINVAL, "out is NULL");
  *out = nullptr;
  int rc = validate(cfg, tensors, n);
  if (rc != ADAMW4_OK) return rc;

  adamw4_handle* h = new (std::nothrow) adamw4_handle();
  if (h == nullptr) return fail(nullptr, ADAMW4_ENOMEM, "host allocation failed");
  h->device = device;
  h->cfg = *cfg;
  build_tables(&h->tabs);
  if (!tables_ok(h->tabs)) {
    delete h;
    return fail(nullptr, ADAMW4_EINVAL, "NF4 bucket table has two midpoints in one bucket");
  }

  // Classify and lay out the state.
  int64_t unit = 0;
  std::vector<DevTensor> dev(std::max(n, 1));
  for (int i = 0; i < n; ++i) {
    HostTensor ht{};
    ht.desc = tensors[i];
    ht.fp32 = fp32_state(tensors[i]);
    if (tensors[i].flags & ADAMW4_T_BF16_PARAM) h->bf16w = true;
    ht.nblocks = (tensors[i].numel + kBlock - 1) / kBlock;
    if (ht.fp32) {
      ht.state_off = h->nfp32;
      h->nfp32 += ht.nblocks * kBlock;     // 512-byte aligned start per tensor
    } else {
      ht.state_off = h->nblocks4;
      h->nblocks4 += ht.nblocks;
    }
    dev[i] = dev_tensor(tensors[i], ht.fp32, unit, ht.state_off);
    ht.unit_begin = unit;
    unit += ht.nblocks;
    h->tensors.push_back(ht);
  }
  h->nunits = unit;

  if (const char* f = std::getenv("ADAMW4_FAIL_ALLOC")) {
    if (f[0] == '1') {
      delete h;
      return fail(nullptr, ADAMW4_ENOMEM, "allocation failure injected by ADAMW4_FAIL_ALLOC");
    }
  }

  DeviceGuard dg(device);
  if (!dg.ok) {
    const cudaError_t e = dg.err;
    delete h;
    return cuda_fail(nullptr, e, "selecting the device");
  }
  // Arena: m codes | v codes | m scales | v scales | fp32 m | fp32 v.
  const size_t codes = (size_t)h->nblocks4 * (kBlock / 2);
  const size_t scales = (size_t)h->nblocks4 * sizeof(float);
  const size_t fp = (size_t)h->nfp32 * sizeof(float);
  size_t off = 0;
  const size_t o_mc = off; off = align_up(off + codes, 256);
  const size_t o_vc = off; off = align_up(off + codes, 256);
  const size_t o_ms = off; off = align_up(off + scales, 256);
  const size_t o_vs = off; off = align_up(off + scales, 256);
  const size_t o_fm = off; off = align_up(off + fp, 256);
  const size_t o_fv = off; off = align_up(off + fp, 256);
  const size_t o_st = off; off = align_up(off + sizeof(uint32_t), 256);
  h->arena_bytes = off;
  cudaError_t e = cudaMalloc(&h->d_arena, h->arena_bytes);
  if (e != cudaSuccess) {
    delete h;
    return fail(nullptr, ADAMW4_ENOMEM, std::string("state allocation: ") + cudaGetErrorString(e));
  }
  e = cudaMalloc(&h->d_tensors, sizeof(DevTensor) * dev.size());
  if (e != cudaSuccess) {
    release(h);
    delete h;
    return fail(nullptr, ADAMW4_ENOMEM, std::string("table allocation: ") + cudaGetErrorString(e));
  }
  uint8_t* base = static_cast<uint8_t*>(h->d_arena);
  h->st.mcodes = base + o_mc;
  h->st.vcodes = base + o_vc;
  h->st.mscale = reinterpret_cast<float*>(base + o_ms);
  h->st.vscale = reinterpret_cast<float*>(base + o_vs);
  h->st.fm = reinterpret_cast<float*>(base + o_fm);
  h->st.fv = reinterpret_cast<float*>(base + o_fv);
  h->d_status = reinterpret_cast<uint32_t*>(base + o_st);
  if ((e = cudaMemset(h->d_arena, 0, h->arena_bytes)) != cudaSuccess ||
      (e = cudaMemcpy(h->d_tensors, dev.data(), sizeof(DevTensor) * dev.size(),
                      cudaMemcpyHostToDevice)) != cudaSuccess) {
    release(h);
    delete h;
    return cuda_fail(nullptr, e, "initialising the state");
  }
  int ge = grid_for(cfg->vcode, h->bf16w, device, &h->grid);
  if (ge != 0) {
    release(h);
    delete h;
    return cuda_fail(nullptr, (cudaError_t)ge, "occupancy query");
  }
  {
    std::lock_guard<std::mutex> lk(g_mu);
    g_live.insert(h);
  }
  *out = h;
  return ADAMW4_OK;
}

extern "C" int adamw4_step(adamw4_handle* h, float lr, void* cuda_stream) {
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  if (!(lr >= 0.0f) || !std::isfinite(lr))
    return fail(h, ADAMW4_EINVAL, "lr must be finite and non-negative");
  DeviceGuard dg(h->device);
  if (!dg.ok) return cuda_fail(h, dg.err, "selecting the device");
  const int64_t t = h->t + 1;
  const StepArgs a = make_args(h->cfg, lr, t);
  const int rc = launch(h, a, static_cast<cudaStream_t>(cuda_stream), 0, h->nunits);
  if (rc != ADAMW4_OK) return rc;
  h->t = t;
  return ADAMW4_OK;
}

extern "C" int adamw4_step_host(adamw4_handle* h, float lr, const uint16_t* const* grads_host,
                                float* const* params_host, void* cuda_stream) {
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  if (!(lr >= 0.0f) || !std::isfinite(lr))
    return fail(h, ADAMW4_EINVAL, "lr must be finite and non-negative");
  for (size_t i = 0; i < h->tensors.size(); ++i) {
    if (grads_host != nullptr && grads_host[i] == nullptr)
      return fail(h, ADAMW4_EINVAL, "grads_host entry is NULL");
    if (params_host != nullptr && params_host[i] == nullptr)
      return fail(h, ADAMW4_EINVAL, "params_host entry is NULL");
  }
  DeviceGuard dg(h->device);
  if (!dg.ok) return cuda_fail(h, dg.err, "selecting the device");
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e;
  const int64_t chunk = host_chunk_units();
  const int64_t nchunks = (h->nunits + chunk - 1) / chunk;
  if (h->s_in == nullptr) {
    if ((e = cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(h, e, "creating the copy streams");
  }
  while ((int64_t)h->events.size() < 2 * nchunks + 2) {
    cudaEvent_t ev;
    if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_fail(h, e, "creating events");
    h->events.push_back(ev);
  }
  const int64_t t = h->t + 1;
  const StepArgs a = make_args(h->cfg, lr, t);
  // The copies wait for the caller's earlier work on the buffers.
  cudaEvent_t ev_start = h->events[2 * nchunks], ev_end = h->events[2 * nchunks + 1];
  if ((e = cudaEventRecord(ev_start, s)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(h->s_in, ev_start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(h->s_out, ev_start, 0)) != cudaSuccess)
    return cuda_fail(h, e, "ordering the copy streams");
  // Piece k: its grads go up on s_in, it steps on the caller's stream, its
  // weights come down on s_out; piece k+1's grads go up meanwhile.
  size_t first = 0;   // first tensor that can reach into the current piece
  for (int64_t k = 0; k < nchunks; ++k) {
    const int64_t u0 = k * chunk, u1 = std::min(h->nunits, u0 + chunk);
    while (first < h->tensors.size() &&
           h->tensors[first].unit_begin + h->tensors[first].nblocks <= u0)
      ++first;
    // copies of the values of piece k, tensor by tensor
    auto copy_piece = [&](bool up) -> cudaError_t {
      for (size_t i = first; i < h->tensors.size() && h->tensors[i].unit_begin < u1; ++i) {
        const HostTensor& ht = h->tensors[i];
        const adamw4_tensor& d = ht.desc;
        const int64_t v0 = (std::max(u0, ht.unit_begin) - ht.unit_begin) * kBlock;
        const int64_t v1 = std::min(
            (std::min(u1, ht.unit_begin + ht.nblocks) - ht.unit_begin) * (int64_t)kBlock, d.numel);
        if (v1 <= v0) continue;
        cudaError_t ce;
        if (up) {
          ce = cudaMemcpyAsync(const_cast<uint16_t*>(d.grad_bf16) + v0, grads_host[i] + v0,
                               (size_t)(v1 - v0) * sizeof(uint16_t), cudaMemcpyHostToDevice,
                               h->s_in);
        } else {
          const size_t wb = param_bytes(d);
          ce = cudaMemcpyAsync(reinterpret_cast<uint8_t*>(params_host[i]) + v0 * wb,
                               reinterpret_cast<const uint8_t*>(d.param) + v0 * wb,
                               (size_t)(v1 - v0) * wb, cudaMemcpyDeviceToHost, h->s_out);
        }
        if (ce != cudaSuccess) return ce;
      }
      return cudaSuccess;
    };
    if (grads_host != nullptr) {
      if ((e = copy_piece(true)) != cudaSuccess) return cuda_fail(h, e, "copying grads to the device");
      if ((e = cudaEventRecord(h->events[2 * k], h->s_in)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(s, h->events[2 * k], 0)) != cudaSuccess)
        return cuda_fail(h, e, "ordering the copy streams");
    }
    const int rc = launch(h, a, s, u0, u1);
    if (rc != ADAMW4_OK) return rc;
    if (params_host != nullptr) {
      if ((e = cudaEventRecord(h->events[2 * k + 1], s)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(h->s_out, h->events[2 * k + 1], 0)) != cudaSuccess)
        return cuda_fail(h, e, "ordering the copy streams");
      if ((e = copy_piece(false)) != cudaSuccess) return cuda_fail(h, e, "copying params to the host");
    }
  }
  if ((e = cudaEventRecord(ev_end, h->s_out)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(s, ev_end, 0)) != cudaSuccess)
    return cuda_fail(h, e, "ordering the copy streams");
  h->t = t;
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(h, e, "synchronising the stream");
  return ADAMW4_OK;
}

extern "C" int adamw4_destroy(adamw4_handle* h) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (h == nullptr || g_live.erase(h) == 0)
      return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  }
  DeviceGuard dg(h->device);
  if (dg.ok) cudaDeviceSynchronize();
  release(h);
  delete h;
  return ADAMW4_OK;
}

extern "C" int adamw4_get_step(const adamw4_handle* h, int64_t* t) {
  if (!live(h) || t == nullptr) return fail(nullptr, ADAMW4_EINVAL, "unknown handle or NULL t");
  *t = h->t;
  return ADAMW4_OK;
}

extern "C" int adamw4_set_step(adamw4_handle* h, int64_t t) {
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  if (t < 0) return fail(h, ADAMW4_EINVAL, "t must be >= 0");
  h->t = t;
  return ADAMW4_OK;
}

extern "C" int64_t adamw4_state_bytes(const adamw4_handle* h) {
  if (!live(h)) return -1;
  int64_t b = 0;
  for (const HostTensor& t : h->tensors)
    b += t.fp32 ? t.desc.numel * 8 : t.nblocks * (kBlock + 2 * (int64_t)sizeof(float));
  return b;
}

namespace {

int64_t blob_bytes(const adamw4_handle* h) {
  int64_t b = 40;
  for (const HostTensor& t : h->tensors)
    b += 16 + (t.fp32 ? t.desc.numel * 8 : t.nblocks * (kBlock + 8));
  return b;
}

struct BlobHead {
  char magic[8];
  uint32_t n_tensors;
  uint32_t vcode;
  int64_t t;
  uint64_t seed;
  uint64_t payload_bytes;
};
static_assert(sizeof(BlobHead) == 40, "blob header");

}  // namespace

extern "C" int adamw4_state_export(const adamw4_handle* hc, void* host_buf, int64_t cap,
                                   int64_t* used) {
  if (!live(hc)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  adamw4_handle* h = const_cast<adamw4_handle*>(hc);
  const int64_t need = blob_bytes(h);
  if (used != nullptr) *used = need;
  if (host_buf == nullptr) return ADAMW4_OK;
  if (cap < need) return fail(h, ADAMW4_ERANGE, "buffer too small for the state blob");
  DeviceGuard dg(h->device);
  if (!dg.ok) return cuda_fail(h, dg.err, "selecting the device");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(h, e, "synchronising before export");
  uint8_t* p = static_cast<uint8_t*>(host_buf);
  BlobHead hd{};
  std::memcpy(hd.magic, "ADAMW4S1", 8);
  hd.n_tensors = (uint32_t)h->tensors.size();
  hd.vcode = (uint32_t)h->cfg.vcode;
  hd.t = h->t;
  hd.seed = h->cfg.seed;
  hd.payload_bytes = (uint64_t)(need - 40);
  std::memcpy(p, &hd, 40);
  p += 40;
  for (const HostTensor& t : h->tensors) {
    const uint32_t id = t.desc.tensor_id, kind = t.fp32 ? 1u : 0u;
    const int64_t numel = t.desc.numel;
    std::memcpy(p, &id, 4);
    std::memcpy(p + 4, &kind, 4);
    std::memcpy(p + 8, &numel, 8);
    p += 16;
    struct Part { const void* src; size_t bytes; };
    Part parts[4];
    int np;
    if (t.fp32) {
      parts[0] = {h->st.fm + t.state_off, (size_t)numel * 4};
      parts[1] = {h->st.fv + t.state_off, (size_t)numel * 4};
      np = 2;
    } else {
      parts[0] = {h->st.mcodes + t.state_off * 64, (size_t)t.nblocks * 64};
      parts[1] = {h->st.vcodes + t.state_off * 64, (size_t)t.nblocks * 64};
      parts[2] = {h->st.mscale + t.state_off, (size_t)t.nblocks * 4};
      parts[3] = {h->st.vscale + t.state_off, (size_t)t.nblocks * 4};
      np = 4;
    }
    for (int k = 0; k < np; ++k) {
      e = cudaMemcpy(p, parts[k].src, parts[k].bytes, cudaMemcpyDeviceToHost);
      if (e != cudaSuccess) return cuda_fail(h, e, "copying the state to the host");
      p += parts[k].bytes;
    }
  }
  return ADAMW4_OK;
}

extern "C" int adamw4_state_import(adamw4_handle* h, const void* host_buf, int64_t len) {
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  if (host_buf == nullptr) return fail(h, ADAMW4_EINVAL, "host_buf is NULL");
  if (len != blob_bytes(h)) return fail(h, ADAMW4_ESTATE, "blob size does not match this handle");
  const uint8_t* p = static_cast<const uint8_t*>(host_buf);
  BlobHead hd;
  std::memcpy(&hd, p, 40);
  if (std::memcmp(hd.magic, "ADAMW4S1", 8) != 0) return fail(h, ADAMW4_ESTATE, "bad blob magic");
  if (hd.n_tensors != h->tensors.size() || hd.vcode != (uint32_t)h->cfg.vcode ||
      hd.seed != h->cfg.seed || hd.payload_bytes != (uint64_t)(len - 40) || hd.t < 0)
    return fail(h, ADAMW4_ESTATE, "blob header does not match this handle");
  // Check every tensor record before touching the device.
  const uint8_t* q = p + 40;
  for (const HostTensor& t : h->tensors) {
    uint32_t id, kind;
    int64_t numel;
    std::memcpy(&id, q, 4);
    std::memcpy(&kind, q + 4, 4);
    std::memcpy(&numel, q + 8, 8);
    if (id != t.desc.tensor_id || kind != (t.fp32 ? 1u : 0u) || numel != t.desc.numel)
      return fail(h, ADAMW4_ESTATE, "blob tensor record does not match tensor " + std::to_string(id));
    q += 16 + (t.fp32 ? numel * 8 : t.nblocks * (kBlock + 8));
  }
  DeviceGuard dg(h->device);
  if (!dg.ok) return cuda_fail(h, dg.err, "selecting the device");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(h, e, "synchronising before import");
  q = p + 40;
  for (const HostTensor& t : h->tensors) {
    q += 16;
    struct Part { void* dst; size_t bytes; };
    Part parts[4];
    int np;
    if (t.fp32) {
      parts[0] = {h->st.fm + t.state_off, (size_t)t.desc.numel * 4};
      parts[1] = {h->st.fv + t.state_off, (size_t)t.desc.numel * 4};
      np = 2;
    } else {
      parts[0] = {h->st.mcodes + t.state_off * 64, (size_t)t.nblocks * 64};
      parts[1] = {h->st.vcodes + t.state_off * 64, (size_t)t.nblocks * 64};
      parts[2] = {h->st.mscale + t.state_off, (size_t)t.nblocks * 4};
      parts[3] = {h->st.vscale + t.state_off, (size_t)t.nblocks * 4};
      np = 4;
    }
    for (int k = 0; k < np; ++k) {
      e = cudaMemcpy(parts[k].dst, q, parts[k].bytes, cudaMemcpyHostToDevice);
      if (e != cudaSuccess) return cuda_fail(h, e, "copying the state to the device");
      q += parts[k].bytes;
    }
  }
  h->t = hd.t;
  return ADAMW4_OK;
}

extern "C" int adamw4_sync(adamw4_handle* h, void* cuda_stream) {
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  DeviceGuard dg(h->device);
  if (!dg.ok) return cuda_fail(h, dg.err, "selecting the device");
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(h, e, "synchronising the stream");
  uint32_t status = 0;
  e = cudaMemcpy(&status, h->d_status, sizeof status, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "reading the status word");
  if (status != 0) {
    e = cudaMemset(h->d_status, 0, sizeof status);
    if (e != cudaSuccess) return cuda_fail(h, e, "clearing the status word");
    return fail(h, ADAMW4_ETIMEOUT,
                "a stage wait in the step kernel ran out of time; the step is incomplete");
  }
  return ADAMW4_OK;
}

extern "C" int adamw4_inject_fault(adamw4_handle* h, int fault) {
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  if (fault != 0 && fault != ADAMW4_FAULT_STALL_PIPELINE)
    return fail(h, ADAMW4_EINVAL, "unknown fault");
  h->fault_stall = (fault == ADAMW4_FAULT_STALL_PIPELINE);
  return ADAMW4_OK;
}

extern "C" int adamw4_launch_info(const adamw4_handle* h, int* grid, int* block, int64_t* units) {
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  const int64_t need = (h->nunits + kHalves - 1) / kHalves;
  if (grid) *grid = (int)std::min<int64_t>(h->grid, need);
  if (block) *block = kCtaThreads;
  if (units) *units = h->nunits;
  return ADAMW4_OK;
}

extern "C" const char* adamw4_last_error(const adamw4_handle* h) {
  if (h != nullptr && live(h)) return h->err.c_str();
  return t_err.c_str();
}

// ---------------------------------------------------------------------------
// Allocation-free step
//
// adamw4_step_noalloc runs the same step kernel without allocating device
// memory.  The kernel's own scratch -- the per-tensor descriptor table it walks
// and the status word its bounded waits report to -- lives in the file-scope
// array below: kNoAllocScratchBytes (about 64.3 KB) on every GPU that loads
// this library, held until the process exits.  The caller passes the inputs
// and outputs (params, grads, and the packed state buffers).
// ---------------------------------------------------------------------------
namespace {

constexpr int kNoAllocMaxTensors = ADAMW4_NOALLOC_MAX_TENSORS;
constexpr size_t kNoAllocStatusBytes = 256;   // status word, padded to keep the table aligned
constexpr size_t kNoAllocScratchBytes =
    kNoAllocStatusBytes + sizeof(DevTensor) * (size_t)kNoAllocMaxTensors;
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocDevice {
  bool ready;
  unsigned char* scratch;   // device address of g_noalloc_scratch on this device
  int grid[ADAMW4_V_ZE_FLOOR + 1][2];   // per vcode, without / with bf16 weights
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];
DevTensor g_noalloc_table[kNoAllocMaxTensors];   // host staging of the table

bool na_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The checks adamw4_create makes, written without containers so that nothing
// is allocated (duplicate ids and overlaps by pairwise comparison).
int na_validate(const adamw4_config* cfg, const adamw4_tensor* ts, int n,
                const adamw4_state_buffers* sb, int64_t t, float lr) {
  if (cfg == nullptr || sb == nullptr) return ADAMW4_EINVAL;
  if (!(cfg->beta1 >= 0.0f && cfg->beta1 < 1.0f) || !(cfg->beta2 >= 0.0f && cfg->beta2 < 1.0f))
    return ADAMW4_EINVAL;
  if (!(cfg->eps > 0.0f) || !std::isfinite(cfg->eps)) return ADAMW4_EINVAL;
  if (cfg->vcode < ADAMW4_V_ZIPSR || cfg->vcode > ADAMW4_V_ZE_FLOOR) return ADAMW4_EINVAL;
  if (cfg->total_steps < 0 || t < 1) return ADAMW4_EINVAL;
  if (!(lr >= 0.0f) || !std::isfinite(lr)) return ADAMW4_EINVAL;
  if (n < 0 || (n > 0 && ts == nullptr)) return ADAMW4_EINVAL;
  if (n > kNoAllocMaxTensors) return ADAMW4_ERANGE;
  if (!na_aligned(sb->mcodes, 16) || !na_aligned(sb->vcodes, 16) || !na_aligned(sb->mscale, 4) ||
      !na_aligned(sb->vscale, 4) || !na_aligned(sb->m32, 16) || !na_aligned(sb->v32, 16))
    return ADAMW4_EALIGN;
  for (int i = 0; i < n; ++i) {
    const adamw4_tensor& x = ts[i];
    if (x.param == nullptr || x.grad_bf16 == nullptr || x.numel <= 0 ||
        x.numel > ((int64_t)1 << 40) || !std::isfinite(x.weight_decay) || piece_error(x) != nullptr)
      return ADAMW4_EINVAL;
    if (!na_aligned(x.param, 16) || !na_aligned(x.grad_bf16, 16)) return ADAMW4_EALIGN;
    const uintptr_t p0 = reinterpret_cast<uintptr_t>(x.param),
                    p1 = p0 + (uintptr_t)x.numel * param_bytes(x);
    const uintptr_t g0 = reinterpret_cast<uintptr_t>(x.grad_bf16), g1 = g0 + (uintptr_t)x.numel * 2u;
    if (p0 < g1 && g0 < p1) return ADAMW4_EINVAL;                 // own grad
    for (int k = 0; k < i; ++k) {
      const adamw4_tensor& y = ts[k];
      if (y.tensor_id == x.tensor_id) return ADAMW4_EINVAL;
      const uintptr_t q0 = reinterpret_cast<uintptr_t>(y.param),
                      q1 = q0 + (uintptr_t)y.numel * param_bytes(y);
      const uintptr_t h0 = reinterpret_cast<uintptr_t>(y.grad_bf16), h1 = h0 + (uintptr_t)y.numel * 2u;
      if ((p0 < q1 && q0 < p1) || (p0 < h1 && h0 < p1) || (q0 < g1 && g0 < q1))
        return ADAMW4_EINVAL;                                     // a param overlaps
    }
  }
  return ADAMW4_OK;
}

}  // namespace

extern "C" int adamw4_step_noalloc(const adamw4_config* cfg, const adamw4_tensor* tensors, int n,
                                   const adamw4_state_buffers* state, int64_t t, float lr,
                                   int device, void* cuda_stream) {
  const int rc = na_validate(cfg, tensors, n, state, t, lr);
  if (rc != ADAMW4_OK) return rc;
  if (device < 0 || device >= kNoAllocMaxDevices) return ADAMW4_EINVAL;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  DeviceGuard dg(device);
  if (!dg.ok) return ADAMW4_ECUDA;
  NoAllocDevice& nd = g_noalloc_dev[device];
  if (!nd.ready) {
    // Once per device, with that device current: the device address of the
    // scratch array (its host-side name is only a stand-in), and the launch
    // geometry.
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&nd.scratch), g_noalloc_scratch) !=
        cudaSuccess)
      return ADAMW4_ECUDA;
    for (int vc = ADAMW4_V_ZIPSR; vc <= ADAMW4_V_ZE_FLOOR; ++vc)
      for (int bw = 0; bw < 2; ++bw)
        if (grid_for(vc, bw != 0, device, &nd.grid[vc][bw]) != 0) return ADAMW4_ECUDA;
    nd.ready = true;
  }
  // The table adamw4_create would build, in the same order and layout.
  int64_t unit = 0, blocks4 = 0, elems32 = 0;
  int bf16w = 0;
  for (int i = 0; i < n; ++i) {
    const adamw4_tensor& x = tensors[i];
    const bool fp32 = fp32_state(x);
    if (x.flags & ADAMW4_T_BF16_PARAM) bf16w = 1;
    const int64_t nb = (x.numel + kBlock - 1) / kBlock;
    g_noalloc_table[i] = dev_tensor(x, fp32, unit, fp32 ? elems32 : blocks4);
    if (fp32) elems32 += nb * kBlock; else blocks4 += nb;
    unit += nb;
  }
  if (unit == 0) return ADAMW4_OK;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  uint32_t* status = reinterpret_cast<uint32_t*>(nd.scratch);
  DevTensor* table = reinterpret_cast<DevTensor*>(nd.scratch + kNoAllocStatusBytes);
  // The array keeps the previous call's contents: clear the status word and
  // overwrite the table.  The copy is from pageable memory, so the staging
  // buffer is free again when the call returns.
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return ADAMW4_ECUDA;
  if (cudaMemcpyAsync(table, g_noalloc_table, sizeof(DevTensor) * (size_t)n,
                      cudaMemcpyHostToDevice, s) != cudaSuccess)
    return ADAMW4_ECUDA;
  CodeTables tabs;
  build_tables(&tabs);
  StepArgs a = make_args(*cfg, lr, t);
  a.status = status;
  a.fault_stall = 0;
  StateArena st;
  st.mcodes = state->mcodes;
  st.vcodes = state->vcodes;
  st.mscale = state->mscale;
  st.vscale = state->vscale;
  st.fm = state->m32;
  st.fv = state->v32;
  const int64_t need = (unit + kHalves - 1) / kHalves;
  launch_vcode(cfg->vcode, bf16w, (int)std::min<int64_t>(nd.grid[cfg->vcode][bf16w], need), s,
               table, 0, unit, a, tabs, st);
  return cudaGetLastError() == cudaSuccess ? ADAMW4_OK : ADAMW4_ECUDA;
}
