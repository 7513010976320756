// adamw4.cu -- fused 4-bit AdamW optimizer step (ZIP-SR / ZE-EDEN) for B200
// (sm_100a), and the C ABI declared in include/adamw4.h.
//
// One kernel launch per step covers every parameter tensor.  The work is a flat
// list of 128-value units: each block of a 4-bit tensor is one unit, and each
// fp32-state tensor is cut into 128-element chunks.  A half-warp owns one unit
// (16 lanes x 8 contiguous values), so a lane moves two 16-byte fp32 weight
// vectors, one 16-byte bf16 gradient vector and one 32-bit word of codes per
// moment.  The grid is persistent (SM count x resident CTAs) and half-warps
// stride through the unit list, which keeps all SMs streaming one contiguous
// window of HBM.
//
// Per unit, following the method flowchart of "ZIP-SR / ZE-EDEN: 4-bit AdamW
// state quantization" (daiwk.github.io, Method): decode the prior moments,
// update them, update the weights, requantise (ZIP-SR or ZE-EDEN for v, NF4 for
// m), pack.  The weights use the unquantised working moments (same page, Core
// equation: weights are updated before the moments are quantised).
//
// Arithmetic follows one fixed binary32 evaluation order with IEEE division
// and square root (__fdiv_rn, __fsqrt_rn) and fused multiply-add only where
// __fmaf_rn is written; the file is built with -fmad=false so nothing else is
// contracted.  With that, codes, scales and weights are reproducible bit for bit
// by any IEEE implementation of the same order.
//
// No tensor cores: the step is a streaming codec, bound by HBM bandwidth.

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

constexpr int kBlock = ADAMW4_BLOCK;        // values per quantisation block
constexpr int kLanesPerUnit = 16;           // a half-warp per block
constexpr int kPerLane = kBlock / kLanesPerUnit;  // 8 values per lane
constexpr int kThreads = 256;               // threads per CTA
constexpr int kVZip = ADAMW4_V_ZIPSR;
constexpr int kVZe = ADAMW4_V_ZEEDEN;
constexpr uint32_t kKindFp32 = 1u << 16;    // internal flag: fp32-state tensor
constexpr uint32_t kStreamV = 0u;           // Philox stream of the v draw
constexpr uint32_t kStreamM = 1u;           // Philox stream of the LM-head m draw

// Philox4x32-10 round multipliers and key increments (Salmon et al., SC'11).
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
  uint32_t pad_;
};
static_assert(sizeof(DevTensor) == 64, "DevTensor layout");

// Per-step scalars, formed on the host in binary64 and rounded once.
struct StepArgs {
  float step_size;   // lr / (1 - b1^t)
  float rs_bc2;      // 1 / sqrt(1 - b2^t)
  float b1, omb1, b2, omb2, eps, lr;
  uint32_t key0, key1;   // Philox key = seed
  uint32_t t_lo;         // step, low word (Philox counter word 2)
  int lm_sr_active;      // final-10% LM-head phase
};

// Code tables, passed by value and staged in shared memory by each CTA.
struct CodeTables {
  float nf4[16];        // NF4 levels, ascending
  float nf4_gap[16];    // nf4[j+1] - nf4[j]
  float vz[16];         // ZIP-SR code points k/15
  float vz_sqrt[16];    // sqrt(k/15)
  float2 rtn[65];       // NF4 nearest-level buckets: .x threshold, .y base code (int bits)
};

struct StateArena {
  uint8_t* mcodes;   // 64 bytes per block, element 2i in the low nibble of byte i
  uint8_t* vcodes;
  float* mscale;     // one per block
  float* vscale;
  float* fm;         // fp32-state tensors
  float* fv;
};

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += kPhiloxW0;
      k1 += kPhiloxW1;
    }
    const uint32_t hi0 = __umulhi(kPhiloxM0, c.x), lo0 = kPhiloxM0 * c.x;
    const uint32_t hi1 = __umulhi(kPhiloxM1, c.z), lo1 = kPhiloxM1 * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// Uniform in [0,1): the top 23 bits of a word times 2^-23 (exact).
__device__ __forceinline__ float uniform23(uint32_t w) {
  return __fsub_rn(__uint_as_float((w >> 9) | 0x3F800000u), 1.0f);
}

// The eight draws of one lane: elements q*4 .. q*4+7 (q = first quad).
__device__ __forceinline__ void draws8(const StepArgs& a, uint32_t tensor_id, uint32_t stream,
                                       uint64_t quad, float u[8]) {
  const uint32_t c3 = tensor_id * 2u + stream;
  const uint4 r0 = philox4x32_10(make_uint4((uint32_t)quad, (uint32_t)(quad >> 32), a.t_lo, c3),
                                 a.key0, a.key1);
  const uint64_t q1 = quad + 1;
  const uint4 r1 = philox4x32_10(make_uint4((uint32_t)q1, (uint32_t)(q1 >> 32), a.t_lo, c3),
                                 a.key0, a.key1);
  u[0] = uniform23(r0.x); u[1] = uniform23(r0.y); u[2] = uniform23(r0.z); u[3] = uniform23(r0.w);
  u[4] = uniform23(r1.x); u[5] = uniform23(r1.y); u[6] = uniform23(r1.z); u[7] = uniform23(r1.w);
}

__device__ __forceinline__ float bf16lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

__device__ __forceinline__ float hmax16(float v, unsigned mask) {
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(mask, v, off));
  return v;
}

// Balanced pairwise sum over the half-warp: partner offsets 1, 2, 4, 8 join
// adjacent 8-value groups in index order (IEEE addition is commutative, so
// both partners hold the same bits).
__device__ __forceinline__ float hsum16_tree(float v, unsigned mask) {
#pragma unroll
  for (int off = 1; off < 16; off <<= 1) v = __fadd_rn(v, __shfl_xor_sync(mask, v, off));
  return v;
}

// NF4 nearest level: #{j : x > mid[j]} through 65 uniform buckets of x.
__device__ __forceinline__ uint32_t nf4_rtn(float x, const float2* rtn) {
  int b = __float_as_int(__fmaf_rn(x, 32.0f, 12582944.0f)) - 0x4B400000;
  b = min(max(b, 0), 64);
  const float2 e = rtn[b];
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

// ---------------------------------------------------------------------------
// The step kernel
// ---------------------------------------------------------------------------

template <int VCODE>
__global__ void __launch_bounds__(kThreads)
adamw4_step_kernel(const DevTensor* __restrict__ tensors, int64_t nunits, StepArgs a,
                   CodeTables tabs, StateArena st) {
  __shared__ float s_nf4[16], s_gap[16], s_vz[16], s_vzs[16];
  __shared__ float2 s_rtn[65];
  if (threadIdx.x < 16) {
    s_nf4[threadIdx.x] = tabs.nf4[threadIdx.x];
    s_gap[threadIdx.x] = tabs.nf4_gap[threadIdx.x];
    s_vz[threadIdx.x] = tabs.vz[threadIdx.x];
    s_vzs[threadIdx.x] = tabs.vz_sqrt[threadIdx.x];
  }
  if (threadIdx.x < 65) s_rtn[threadIdx.x] = tabs.rtn[threadIdx.x];
  __syncthreads();

  const int lane = threadIdx.x & 15;
  const unsigned hmask = 0xFFFFu << (threadIdx.x & 16);
  const int64_t H = (int64_t)gridDim.x * (kThreads / kLanesPerUnit);
  int64_t u = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / kLanesPerUnit;

  // Cached descriptor of the current tensor; half-warps move forward only.
  int ti = -1;
  int64_t t_begin = 0, t_end = 0, t_numel = 0, t_soff = 0;
  float* t_param = nullptr;
  const uint16_t* t_grad = nullptr;
  uint32_t t_id = 0, t_flags = 0;
  float decay = 1.0f;

  for (; u < nunits; u += H) {
    if (u >= t_end) {
      do {
        ++ti;
        t_end = __ldg(&tensors[ti].unit_end);
      } while (u >= t_end);
      const DevTensor* d = &tensors[ti];
      t_begin = __ldg(&d->unit_begin);
      t_numel = __ldg(&d->numel);
      t_soff = __ldg(&d->state_off);
      t_param = d->param;
      t_grad = d->grad;
      t_id = __ldg(&d->tensor_id);
      t_flags = __ldg(&d->flags);
      decay = (float)(1.0 - (double)a.lr * (double)__ldg(&d->weight_decay));
    }
    const int64_t ub = u - t_begin;               // unit within the tensor
    const int64_t e0 = ub * kBlock;               // its first element
    const int nvalid = (int)min((int64_t)kBlock, t_numel - e0);
    const int my0 = lane * kPerLane;
    const int myn = min(max(nvalid - my0, 0), kPerLane);
    float* wp = t_param + e0 + my0;
    const uint16_t* gp = t_grad + e0 + my0;

    // ---- load weights and gradients ----
    float w[kPerLane];
    float g[kPerLane];
    if (myn == kPerLane) {
      const float4 wa = *reinterpret_cast<const float4*>(wp);
      const float4 wb = *reinterpret_cast<const float4*>(wp + 4);
      const uint4 gg = *reinterpret_cast<const uint4*>(gp);
      w[0] = wa.x; w[1] = wa.y; w[2] = wa.z; w[3] = wa.w;
      w[4] = wb.x; w[5] = wb.y; w[6] = wb.z; w[7] = wb.w;
      g[0] = bf16lo(gg.x); g[1] = bf16hi(gg.x); g[2] = bf16lo(gg.y); g[3] = bf16hi(gg.y);
      g[4] = bf16lo(gg.z); g[5] = bf16hi(gg.z); g[6] = bf16lo(gg.w); g[7] = bf16hi(gg.w);
    } else {
#pragma unroll
      for (int i = 0; i < kPerLane; ++i) {
        w[i] = (i < myn) ? wp[i] : 0.0f;
        g[i] = (i < myn) ? __uint_as_float((uint32_t)gp[i] << 16) : 0.0f;
      }
    }

    if (t_flags & kKindFp32) {
      // ---- fp32-state AdamW chunk ----
      float* mp = st.fm + t_soff + e0 + my0;
      float* vp = st.fv + t_soff + e0 + my0;
      float m[kPerLane], v[kPerLane];
      if (myn == kPerLane) {
        const float4 ma = *reinterpret_cast<const float4*>(mp);
        const float4 mb = *reinterpret_cast<const float4*>(mp + 4);
        const float4 va = *reinterpret_cast<const float4*>(vp);
        const float4 vb = *reinterpret_cast<const float4*>(vp + 4);
        m[0] = ma.x; m[1] = ma.y; m[2] = ma.z; m[3] = ma.w;
        m[4] = mb.x; m[5] = mb.y; m[6] = mb.z; m[7] = mb.w;
        v[0] = va.x; v[1] = va.y; v[2] = va.z; v[3] = va.w;
        v[4] = vb.x; v[5] = vb.y; v[6] = vb.z; v[7] = vb.w;
      } else {
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
          m[i] = (i < myn) ? mp[i] : 0.0f;
          v[i] = (i < myn) ? vp[i] : 0.0f;
        }
      }
#pragma unroll
      for (int i = 0; i < kPerLane; ++i) {
        const float m1 = __fmaf_rn(a.b1, m[i], __fmul_rn(a.omb1, g[i]));
        const float v1 = __fmaf_rn(a.b2, v[i], __fmul_rn(a.omb2, __fmul_rn(g[i], g[i])));
        const float den = __fmaf_rn(__fsqrt_rn(v1), a.rs_bc2, a.eps);
        w[i] = __fmaf_rn(-a.step_size, __fdiv_rn(m1, den), __fmul_rn(w[i], decay));
        m[i] = m1;
        v[i] = v1;
      }
      if (myn == kPerLane) {
        *reinterpret_cast<float4*>(wp) = make_float4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<float4*>(wp + 4) = make_float4(w[4], w[5], w[6], w[7]);
        *reinterpret_cast<float4*>(mp) = make_float4(m[0], m[1], m[2], m[3]);
        *reinterpret_cast<float4*>(mp + 4) = make_float4(m[4], m[5], m[6], m[7]);
        *reinterpret_cast<float4*>(vp) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4*>(vp + 4) = make_float4(v[4], v[5], v[6], v[7]);
      } else {
#pragma unroll
        for (int i = 0; i < kPerLane; ++i)
          if (i < myn) { wp[i] = w[i]; mp[i] = m[i]; vp[i] = v[i]; }
      }
      continue;
    }

    // ---- 4-bit block: load codes and scales ----
    const int64_t blk = t_soff + ub;
    uint32_t* mcw = reinterpret_cast<uint32_t*>(st.mcodes + blk * (kBlock / 2)) + lane;
    uint32_t* vcw = reinterpret_cast<uint32_t*>(st.vcodes + blk * (kBlock / 2)) + lane;
    const uint32_t mc = *mcw;
    const uint32_t vc = *vcw;
    const float sm = st.mscale[blk];
    const float sv = st.vscale[blk];

    // ---- decode, moment update, weight update ----
    float m1[kPerLane], v1[kPerLane], den[kPerLane];
    float am = 0.0f, av = 0.0f;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const float m0 = __fmul_rn(s_nf4[(mc >> (4 * i)) & 15u], sm);
      const uint32_t cv = (vc >> (4 * i)) & 15u;
      const float q0 = (VCODE == kVZip) ? s_vz[cv] : __fmul_rn((float)(cv + 1), 0.0625f);
      const float v0 = __fmul_rn(q0, sv);
      m1[i] = __fmaf_rn(a.b1, m0, __fmul_rn(a.omb1, g[i]));
      v1[i] = __fmaf_rn(a.b2, v0, __fmul_rn(a.omb2, __fmul_rn(g[i], g[i])));
      den[i] = __fmaf_rn(__fsqrt_rn(v1[i]), a.rs_bc2, a.eps);
      w[i] = __fmaf_rn(-a.step_size, __fdiv_rn(m1[i], den[i]), __fmul_rn(w[i], decay));
      if (i < myn) {
        am = fmaxf(am, fabsf(m1[i]));
        av = fmaxf(av, v1[i]);
      }
    }
    if (myn == kPerLane) {
      *reinterpret_cast<float4*>(wp) = make_float4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<float4*>(wp + 4) = make_float4(w[4], w[5], w[6], w[7]);
    } else {
#pragma unroll
      for (int i = 0; i < kPerLane; ++i)
        if (i < myn) wp[i] = w[i];
    }
    am = hmax16(am, hmask);
    av = hmax16(av, hmask);

    // ---- first moment: absmax scale, NF4 codes ----
    uint32_t mco = 0;
    float mso = 0.0f;
    if (am >= FLT_MIN) {
      const float inv = __fdiv_rn(1.0f, am);
      if ((t_flags & ADAMW4_T_LM_HEAD) && a.lm_sr_active) {
        float ud[kPerLane];
        draws8(a, t_id, kStreamM, (uint64_t)(e0 + my0) >> 2, ud);
#pragma unroll
        for (int i = 0; i < kPerLane; ++i)
          if (i < myn) mco |= nf4_sr(__fmul_rn(m1[i], inv), ud[i], s_nf4, s_gap) << (4 * i);
      } else {
#pragma unroll
        for (int i = 0; i < kPerLane; ++i)
          if (i < myn) mco |= nf4_rtn(__fmul_rn(m1[i], inv), s_rtn) << (4 * i);
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
        float ud[kPerLane];
        draws8(a, t_id, kStreamV, (uint64_t)(e0 + my0) >> 2, ud);
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
          if (i < myn) {
            const float x = __fmul_rn(v1[i], inv);
            int k = min(__float2int_rz(__fmul_rn(x, 15.0f)), 14);
            if (x < s_vz[k]) --k;
            else if (k < 14 && x >= s_vz[k + 1]) ++k;
            const float da = __fmaf_rn(s_vzs[k], R, a.eps);
            const float db = __fmaf_rn(s_vzs[k + 1], R, a.eps);
            bool lower;
            if (da == db) {
              lower = __fmul_rn(ud[i], __fsub_rn(s_vz[k + 1], s_vz[k])) < __fsub_rn(s_vz[k + 1], x);
            } else {
              lower = __fmul_rn(ud[i], __fmul_rn(__fsub_rn(db, da), den[i])) <
                      __fmul_rn(__fsub_rn(db, den[i]), da);
            }
            vco |= (uint32_t)(lower ? k : k + 1) << (4 * i);
          }
        }
        vso = av;
      } else {
        // ZE-EDEN ("ZIP-SR / ZE-EDEN", Core equation): nearest zero-excluded
        // code point, scale times ||x||^2 / max(<x,Q(x)>, 1e-12 s^2) on x = v/s.
        float xx[kPerLane], xq[kPerLane];
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
          const float x = __fmul_rn(v1[i], inv);
          int k = __float2int_rz(rintf(__fmul_rn(x, 16.0f))) - 1;
          k = min(max(k, 0), 15);
          const float q = __fmul_rn((float)(k + 1), 0.0625f);
          const bool ok = i < myn;
          xx[i] = ok ? __fmul_rn(x, x) : 0.0f;
          xq[i] = ok ? __fmul_rn(x, q) : 0.0f;
          if (ok) vco |= (uint32_t)k << (4 * i);
        }
        float sxx = __fadd_rn(__fadd_rn(__fadd_rn(xx[0], xx[1]), __fadd_rn(xx[2], xx[3])),
                              __fadd_rn(__fadd_rn(xx[4], xx[5]), __fadd_rn(xx[6], xx[7])));
        float sxq = __fadd_rn(__fadd_rn(__fadd_rn(xq[0], xq[1]), __fadd_rn(xq[2], xq[3])),
                              __fadd_rn(__fadd_rn(xq[4], xq[5]), __fadd_rn(xq[6], xq[7])));
        sxx = hsum16_tree(sxx, hmask);
        sxq = hsum16_tree(sxq, hmask);
        vso = __fmul_rn(av, __fdiv_rn(sxx, fmaxf(sxq, 1e-12f)));
      }
    }

    // ---- pack and store ----
    *mcw = mco;
    *vcw = vco;
    if (lane == 0) {
      st.mscale[blk] = mso;
      st.vscale[blk] = vso;
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
  int grid = 0;
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
  // Midpoints of adjacent binary32 levels, exact in binary64, rounded once.
  float mid[15];
  for (int j = 0; j < 15; ++j)
    mid[j] = (float)(((double)kNF4Levels[j] + (double)kNF4Levels[j + 1]) * 0.5);
  // Bucket b of x is round(32 x + 32) clamped to [0, 64] (monotone in x).  A
  // bucket holds at most one midpoint, so the nearest level is the count of
  // midpoints in lower buckets plus one comparison.
  int bucket_of[15];
  for (int j = 0; j < 15; ++j) {
    const float y = std::fma(mid[j], 32.0f, 12582944.0f);
    int32_t bits;
    std::memcpy(&bits, &y, 4);
    bucket_of[j] = std::min(std::max(bits - 0x4B400000, 0), 64);
  }
  for (int b = 0; b < 65; ++b) {
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
  a.key0 = (uint32_t)c.seed;
  a.key1 = (uint32_t)(c.seed >> 32);
  a.t_lo = (uint32_t)t;
  a.lm_sr_active = (c.total_steps > 0) && (10 * t > 9 * c.total_steps);
  return a;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate(const adamw4_config* cfg, const adamw4_tensor* ts, int n) {
  if (cfg == nullptr) return fail(nullptr, ADAMW4_EINVAL, "config is NULL");
  if (!(cfg->beta1 >= 0.0f && cfg->beta1 < 1.0f) || !(cfg->beta2 >= 0.0f && cfg->beta2 < 1.0f))
    return fail(nullptr, ADAMW4_EINVAL, "beta1 and beta2 must lie in [0, 1)");
  if (!(cfg->eps > 0.0f) || !std::isfinite(cfg->eps))
    return fail(nullptr, ADAMW4_EINVAL, "eps must be positive and finite");
  if (!(cfg->lr >= 0.0f) || !std::isfinite(cfg->lr))
    return fail(nullptr, ADAMW4_EINVAL, "lr must be finite and non-negative");
  if (cfg->vcode != ADAMW4_V_ZIPSR && cfg->vcode != ADAMW4_V_ZEEDEN)
    return fail(nullptr, ADAMW4_EINVAL, "vcode must be ADAMW4_V_ZIPSR or ADAMW4_V_ZEEDEN");
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
    if (!ids.insert(t.tensor_id).second)
      return fail(nullptr, ADAMW4_EINVAL, at + "duplicate tensor_id " + std::to_string(t.tensor_id));
    const uintptr_t p = reinterpret_cast<uintptr_t>(t.param);
    const uintptr_t g = reinterpret_cast<uintptr_t>(t.grad_bf16);
    ranges.push_back({p, p + (uintptr_t)t.numel * 4u, i, true});
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

template <int VCODE>
int occupancy_grid(int device, int* grid) {
  int sms = 0, per_sm = 0;
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) return (int)e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, adamw4_step_kernel<VCODE>,
                                                    kThreads, 0);
  if (e != cudaSuccess) return (int)e;
  *grid = sms * std::max(per_sm, 1);
  return 0;
}

int launch(adamw4_handle* h, const StepArgs& a, cudaStream_t s) {
  if (h->nunits == 0) return ADAMW4_OK;
  const int64_t need = (h->nunits + (kThreads / kLanesPerUnit) - 1) / (kThreads / kLanesPerUnit);
  const int grid = (int)std::min<int64_t>(h->grid, need);
  if (h->cfg.vcode == kVZip)
    adamw4_step_kernel<kVZip><<<grid, kThreads, 0, s>>>(h->d_tensors, h->nunits, a, h->tabs, h->st);
  else
    adamw4_step_kernel<kVZe><<<grid, kThreads, 0, s>>>(h->d_tensors, h->nunits, a, h->tabs, h->st);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(h, e, "step kernel launch");
  return ADAMW4_OK;
}

void release(adamw4_handle* h) {
  if (h->d_tensors) cudaFree(h->d_tensors);
  if (h->d_arena) cudaFree(h->d_arena);
  h->d_tensors = nullptr;
  h->d_arena = nullptr;
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
    ht.fp32 = tensors[i].numel < ADAMW4_MIN_QUANT_NUMEL ||
              (tensors[i].flags & (ADAMW4_T_NORM | ADAMW4_T_FP32_STATE)) != 0;
    ht.nblocks = (tensors[i].numel + kBlock - 1) / kBlock;
    if (ht.fp32) {
      ht.state_off = h->nfp32;
      h->nfp32 += ht.nblocks * kBlock;     // 512-byte aligned start per tensor
    } else {
      ht.state_off = h->nblocks4;
      h->nblocks4 += ht.nblocks;
    }
    DevTensor& d = dev[i];
    d.param = tensors[i].param;
    d.grad = tensors[i].grad_bf16;
    d.numel = tensors[i].numel;
    d.unit_begin = unit;
    d.unit_end = unit + ht.nblocks;
    d.state_off = ht.state_off;
    d.tensor_id = tensors[i].tensor_id;
    d.flags = tensors[i].flags | (ht.fp32 ? kKindFp32 : 0u);
    d.weight_decay = tensors[i].weight_decay;
    d.pad_ = 0;
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
  h->arena_bytes = std::max<size_t>(off, 256);
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
  if ((e = cudaMemset(h->d_arena, 0, h->arena_bytes)) != cudaSuccess ||
      (e = cudaMemcpy(h->d_tensors, dev.data(), sizeof(DevTensor) * dev.size(),
                      cudaMemcpyHostToDevice)) != cudaSuccess) {
    release(h);
    delete h;
    return cuda_fail(nullptr, e, "initialising the state");
  }
  int ge = (cfg->vcode == kVZip) ? occupancy_grid<kVZip>(device, &h->grid)
                                 : occupancy_grid<kVZe>(device, &h->grid);
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
  const int rc = launch(h, a, static_cast<cudaStream_t>(cuda_stream));
  if (rc != ADAMW4_OK) return rc;
  h->t = t;
  return ADAMW4_OK;
}

extern "C" int adamw4_step_host(adamw4_handle* h, float lr, const uint16_t* const* grads_host,
                                float* const* params_host, void* cuda_stream) {
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  DeviceGuard dg(h->device);
  if (!dg.ok) return cuda_fail(h, dg.err, "selecting the device");
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e;
  if (grads_host != nullptr) {
    for (size_t i = 0; i < h->tensors.size(); ++i) {
      const adamw4_tensor& d = h->tensors[i].desc;
      if (grads_host[i] == nullptr) return fail(h, ADAMW4_EINVAL, "grads_host entry is NULL");
      e = cudaMemcpyAsync(const_cast<uint16_t*>(d.grad_bf16), grads_host[i],
                          (size_t)d.numel * sizeof(uint16_t), cudaMemcpyHostToDevice, s);
      if (e != cudaSuccess) return cuda_fail(h, e, "copying grads to the device");
    }
  }
  int rc = adamw4_step(h, lr, cuda_stream);
  if (rc != ADAMW4_OK) return rc;
  if (params_host != nullptr) {
    for (size_t i = 0; i < h->tensors.size(); ++i) {
      const adamw4_tensor& d = h->tensors[i].desc;
      if (params_host[i] == nullptr) return fail(h, ADAMW4_EINVAL, "params_host entry is NULL");
      e = cudaMemcpyAsync(params_host[i], d.param, (size_t)d.numel * sizeof(float),
                          cudaMemcpyDeviceToHost, s);
      if (e != cudaSuccess) return cuda_fail(h, e, "copying params to the host");
    }
  }
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

extern "C" int adamw4_launch_info(const adamw4_handle* h, int* grid, int* block, int64_t* units) {
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  const int64_t need = (h->nunits + (kThreads / kLanesPerUnit) - 1) / (kThreads / kLanesPerUnit);
  if (grid) *grid = (int)std::min<int64_t>(h->grid, need);
  if (block) *block = kThreads;
  if (units) *units = h->nunits;
  return ADAMW4_OK;
}

extern "C" const char* adamw4_last_error(const adamw4_handle* h) {
  if (h != nullptr && live(h)) return h->err.c_str();
  return t_err.c_str();
}
