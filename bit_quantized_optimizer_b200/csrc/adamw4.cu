// adamw4.cu -- the C ABI (include/adamw4.h) of the fused 4-bit AdamW step
// (ZIP-SR / ZE-EDEN) for B200 (sm_100a): validation and classification of the
// tensor list, the state arena, step scalars and code tables, launches (one per
// step, or one per piece of the pipelined host-buffer step), checkpoints, and
// the allocation-free entry point.  The kernel is in adamw4_kernel.cuh.

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>   // header-only; ranges show up under a profiler

#include <algorithm>
#include <atomic>
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
#include "adamw4_kernel.cuh"

namespace {

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

// The NF4 nearest-level bucket of x (the kernel's nf4_rtn_bucket reads the
// same one from the bits of fma(x, 4096, 1.5 * 2^23 + 4096)).
int nf4_bucket(float x) {
  const float y = std::fma(x, 4096.0f, 12587008.0f);
  int32_t bits;
  std::memcpy(&bits, &y, 4);
  return std::min(std::max(bits - 0x4B400000, 0), 8192) >> 7;
}

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
  // Bucket b of x is floor(round(4096 x + 4096) / 128), in [0, 64] for
  // |x| <= 1 + 2^-23 and monotone in x.  A bucket holds at most one midpoint,
  // so the nearest level is the count of midpoints in lower buckets plus one
  // comparison.
  int bucket_of[15];
  for (int j = 0; j < 15; ++j) bucket_of[j] = nf4_bucket(mid[j]);
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

// The shared-memory tables of one code family (zero_excluded: the ZE codes
// (k+1)/16, else the zero-inclusive k/15), as each CTA of the step kernel
// holds them.
void fill_smem_tables(const CodeTables& T, bool zero_excluded, SmemTables* S) {
  for (int t = 0; t < 256; ++t) {
    S->mpair[t] = make_float2(T.nf4[t & 15], T.nf4[t >> 4]);
    const float lo = zero_excluded ? (float)((t & 15) + 1) * 0.0625f : T.vz[t & 15];
    const float hi = zero_excluded ? (float)((t >> 4) + 1) * 0.0625f : T.vz[t >> 4];
    S->vpair[t] = make_float2(lo, hi);
  }
  for (int t = 0; t < 16; ++t) {
    S->nf4[t] = T.nf4[t];
    S->gap[t] = T.nf4_gap[t];
    S->vz[t] = T.vz[t];
    S->zip[t] = make_float4(t == 15 ? INFINITY : T.vz[t], T.vz_sqrt[std::max(t - 1, 0)],
                            T.vz_sqrt[t], T.vz_sqrt[std::min(t + 1, 15)]);
    S->vzp[t] = make_float2(T.vz[t], T.vz[std::min(t + 1, 15)]);
    S->vzmid[t] = T.vz_mid[t];
  }
}

// Writes the code tables into the device's g_code_tables once per device
// (cudaMemcpyToSymbol; no allocation).  The caller has the device current.
std::mutex g_tables_mu;
bool g_tables_ready[64];

cudaError_t upload_tables(int device) {
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_tables_mu);
  if (g_tables_ready[device]) return cudaSuccess;
  CodeTables T;
  build_tables(&T);
  static SmemTables host[2];
  fill_smem_tables(T, false, &host[0]);
  fill_smem_tables(T, true, &host[1]);
  cudaError_t e = cudaMemcpyToSymbol(g_code_tables, host, sizeof host, 0,
                                     cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return e;
  // The lane tables: each entry repeated across the columns of its row.
  static LaneTables lt;
  for (int b = 0; b < 128; ++b)
    for (int c = 0; c < 16; ++c) lt.nf4b[b][c] = T.rtn[b];
  for (int k = 0; k < 16; ++k) {
    for (int c = 0; c < 32; ++c) {
      lt.nf4[k][c] = T.nf4[k];
      lt.vz[k][c] = T.vz[k];
    }
  }
  e = cudaMemcpyToSymbol(g_lane_tables, &lt, sizeof lt, 0, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) g_tables_ready[device] = true;
  return e;
}

bool tables_ok(const CodeTables& T) {
  int seen[65] = {0};
  for (int j = 0; j < 15; ++j) {
    const float mid = (float)(((double)T.nf4[j] + (double)T.nf4[j + 1]) * 0.5);
    if (++seen[nf4_bucket(mid)] > 1) return false;
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
  a.nstep = -a.step_size;
  // Ranges of the kernel's fast square root and division (exact_math.cuh):
  // v1 in [2^-100, 2^64] keeps sqrt(v1) rs_bc2 + eps within [eps, 2^53) when
  // rs_bc2 <= 2^20; |m1| >= 2^-60 keeps the quotient at or above 2^-113 and
  // its remainder exact; |m1| <= 2^100 eps keeps it at or below 2^100.  With
  // eps outside [2^-60, 2^10] or rs_bc2 above 2^20 every lane takes the IEEE
  // operations instead (m_hi < 0).
  a.m_lo = 0x1p-60f;
  a.v_lo = 0x1p-100f;
  a.v_hi = 0x1p64f;
  const bool fast_ok = a.eps >= 0x1p-60f && a.eps <= 0x1p10f && a.rs_bc2 <= 0x1p20f;
  a.m_hi = fast_ok ? std::min(std::ldexp(a.eps, 100), 0x1p100f) : -1.0f;
  auto pair = [](float x) { return make_float2(x, x); };
  a.p_b1 = pair(a.b1);
  a.p_omb1 = pair(a.omb1);
  a.p_nb2 = pair(-a.b2);
  a.p_nomb2 = pair(-a.omb2);
  a.p_rs = pair(a.rs_bc2);
  a.p_eps = pair(a.eps);
  a.p_neps = pair(-a.eps);
  a.p_nstep = pair(a.nstep);
  a.k_half = pair(0.5f);
  a.k_one = pair(1.0f);
  a.k_zero = pair(0.0f);
  a.k_m1 = pair(-1.0f);
  a.k_15 = pair(15.0f);
  a.k_16 = pair(16.0f);
  a.k_4096 = pair(4096.0f);
  a.k_magic = pair(kMagic);
  a.k_magic4096 = pair(kMagic + 4096.0f);
  a.k_nmagic_16 = pair(-kMagic / 16.0f);                 // exact
  a.k_1_16 = pair(0.0625f);
  a.k_2m32 = pair(0x1p-32f);
  // the arithmetic decode of zero-excluded v codes: scales 2^-(p+4) and
  // offsets 1/16 - kMagic 2^-(p+4) for nibbles at bit p = 0, 4 (byte 0) and
  // 8, 12 (byte 1), all exact
  a.k_ze_scale0 = make_float2(0x1p-4f, 0x1p-8f);
  a.k_ze_off0 = make_float2(0.0625f - kMagic * 0x1p-4f, 0.0625f - kMagic * 0x1p-8f);
  a.k_ze_scale1 = make_float2(0x1p-12f, 0x1p-16f);
  a.k_ze_off1 = make_float2(0.0625f - kMagic * 0x1p-12f, 0.0625f - kMagic * 0x1p-16f);
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
  if (cfg->vcode < ADAMW4_V_ZIPSR || cfg->vcode > ADAMW4_V_ZIPSR_U32)
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
    case kVZip32: return occupancy_grid<kVZip32, BF16W>(device, grid);
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
              const StepArgs& a, const StateArena& st) {
  const int n = kCtaThreads;
  const int smem = kSmemStages;
  switch (vcode) {
    case kVZip:
      adamw4_step_kernel<kVZip, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, st);
      break;
    case kVZe:
      adamw4_step_kernel<kVZe, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, st);
      break;
    case kVZiRtn:
      adamw4_step_kernel<kVZiRtn, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, st);
      break;
    case kVZiSr:
      adamw4_step_kernel<kVZiSr, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, st);
      break;
    case kVZeFloor:
      adamw4_step_kernel<kVZeFloor, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, st);
      break;
    default:
      adamw4_step_kernel<kVZip32, BF16W><<<grid, n, smem, s>>>(T, u0, u1, a, st);
      break;
  }
}

// Enqueues the step kernel instantiated for vcode over units [u0, u1) of the
// table; bf16w selects the instantiation that reads and writes bf16 weights
// where a tensor asks for it.
void launch_vcode(int vcode, bool bf16w, int grid, cudaStream_t s, const DevTensor* T,
                  int64_t u0, int64_t u1, const StepArgs& a, const StateArena& st) {
  if (bf16w) launch_w<true>(vcode, grid, s, T, u0, u1, a, st);
  else launch_w<false>(vcode, grid, s, T, u0, u1, a, st);
}

// One launch over units [u0, u1) of the handle's list.
int launch(adamw4_handle* h, StepArgs a, cudaStream_t s, int64_t u0, int64_t u1) {
  if (u1 <= u0) return ADAMW4_OK;
  const int64_t need = (u1 - u0 + kTileUnits - 1) / kTileUnits;
  const int grid = (int)std::min<int64_t>(h->grid, need);
  a.status = h->d_status;
  a.fault_stall = h->fault_stall;
  h->fault_stall = 0;
  launch_vcode(h->cfg.vcode, h->bf16w, grid, s, h->d_tensors, u0, u1, a, h->st);
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
  {
    CodeTables tabs;
    build_tables(&tabs);
    if (!tables_ok(tabs)) {
      delete h;
      return fail(nullptr, ADAMW4_EINVAL, "NF4 bucket table has two midpoints in one bucket");
    }
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
  h->st.nblocks4 = h->nblocks4;
  h->st.n32 = h->nfp32;
  h->st.vs_minus_ms = h->st.vscale - h->st.mscale;
  h->d_status = reinterpret_cast<uint32_t*>(base + o_st);
  if ((e = cudaMemset(h->d_arena, 0, h->arena_bytes)) != cudaSuccess ||
      (e = cudaMemcpy(h->d_tensors, dev.data(), sizeof(DevTensor) * dev.size(),
                      cudaMemcpyHostToDevice)) != cudaSuccess) {
    release(h);
    delete h;
    return cuda_fail(nullptr, e, "initialising the state");
  }
  if ((e = upload_tables(device)) != cudaSuccess) {
    release(h);
    delete h;
    return cuda_fail(nullptr, e, "writing the code tables");
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

// NVTX range for the duration of one ABI call (tracing under nsys / ncu).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

extern "C" int adamw4_step(adamw4_handle* h, float lr, void* cuda_stream) {
  NvtxRange nvtx("adamw4_step");
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
  NvtxRange nvtx("adamw4_step_host");
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

namespace {

// The status code (and message) of a non-zero device status word: a wait
// that ran out first, since it leaves the step incomplete.
int status_error(adamw4_handle* h, uint32_t status) {
  if (status & 1u)
    return fail(h, ADAMW4_ETIMEOUT,
                "a stage wait in the step kernel ran out of time; the step is incomplete");
  if (status & 2u)
    return fail(h, ADAMW4_ECHECK,
                "checked build: a unit's values or state lay outside its tensor or the arena; "
                "that unit was skipped");
  return fail(h, ADAMW4_ENONFINITE,
              "a step produced a non-finite weight (a NaN or infinite grad or weight, or an "
              "overflow); the step ran to the end");
}

}  // namespace

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
    return status_error(h, status);
  }
  return ADAMW4_OK;
}

namespace {
std::atomic<int> g_noalloc_fault_stall{0};   // test hook for the next noalloc call
}  // namespace

extern "C" int adamw4_inject_fault(adamw4_handle* h, int fault) {
  if (fault != 0 && fault != ADAMW4_FAULT_STALL_PIPELINE)
    return fail(live(h) ? h : nullptr, ADAMW4_EINVAL, "unknown fault");
  if (h == nullptr) {   // the next adamw4_step_noalloc call
    g_noalloc_fault_stall.store(fault == ADAMW4_FAULT_STALL_PIPELINE ? 1 : 0);
    return ADAMW4_OK;
  }
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  h->fault_stall = (fault == ADAMW4_FAULT_STALL_PIPELINE);
  return ADAMW4_OK;
}

extern "C" int adamw4_tensor_state_kind(const adamw4_tensor* t) {
  if (t == nullptr || t->numel <= 0 || piece_error(*t) != nullptr) return ADAMW4_EINVAL;
  return fp32_state(*t) ? 1 : 0;
}

extern "C" int adamw4_launch_info(const adamw4_handle* h, int* grid, int* block, int64_t* units) {
  if (!live(h)) return fail(nullptr, ADAMW4_EINVAL, "unknown or destroyed handle");
  const int64_t need = (h->nunits + kTileUnits - 1) / kTileUnits;
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
  int grid[ADAMW4_V_ZIPSR_U32 + 1][2];  // per vcode, without / with bf16 weights
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
  if (cfg->vcode < ADAMW4_V_ZIPSR || cfg->vcode > ADAMW4_V_ZIPSR_U32) return ADAMW4_EINVAL;
  if (cfg->total_steps < 0 || t < 1) return ADAMW4_EINVAL;
  if (!(lr >= 0.0f) || !std::isfinite(lr)) return ADAMW4_EINVAL;
  if (n < 0 || (n > 0 && ts == nullptr)) return ADAMW4_EINVAL;
  if (n > kNoAllocMaxTensors) return ADAMW4_ERANGE;
  if (!na_aligned(sb->mcodes, 16) || !na_aligned(sb->vcodes, 16) || !na_aligned(sb->mscale, 4) ||
      !na_aligned(sb->vscale, 4) || !na_aligned(sb->m32, 16) || !na_aligned(sb->v32, 16))
    return ADAMW4_EALIGN;
  int64_t blocks4 = 0, elems32 = 0;   // what the list needs of each state buffer
  for (int i = 0; i < n; ++i) {
    const adamw4_tensor& x = ts[i];
    if (x.param == nullptr || x.grad_bf16 == nullptr || x.numel <= 0 ||
        x.numel > ((int64_t)1 << 40) || !std::isfinite(x.weight_decay) || piece_error(x) != nullptr)
      return ADAMW4_EINVAL;
    if (!na_aligned(x.param, 16) || !na_aligned(x.grad_bf16, 16)) return ADAMW4_EALIGN;
    if (fp32_state(x)) elems32 += x.numel; else blocks4 += (x.numel + kBlock - 1) / kBlock;
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
  // the state buffers the list uses must be given (a NULL one would be read)
  if (blocks4 > 0 && (sb->mcodes == nullptr || sb->vcodes == nullptr || sb->mscale == nullptr ||
                      sb->vscale == nullptr))
    return ADAMW4_EINVAL;
  if (elems32 > 0 && (sb->m32 == nullptr || sb->v32 == nullptr)) return ADAMW4_EINVAL;
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
    for (int vc = ADAMW4_V_ZIPSR; vc <= ADAMW4_V_ZIPSR_U32; ++vc)
      for (int bw = 0; bw < 2; ++bw)
        if (grid_for(vc, bw != 0, device, &nd.grid[vc][bw]) != 0) return ADAMW4_ECUDA;
    if (upload_tables(device) != cudaSuccess) return ADAMW4_ECUDA;
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
  // The array keeps the previous call's contents: overwrite the table (the
  // status word accumulates until adamw4_noalloc_sync reads and clears it).
  // The copy is from pageable memory, so the staging buffer is free again when
  // the call returns.
  if (cudaMemcpyAsync(table, g_noalloc_table, sizeof(DevTensor) * (size_t)n,
                      cudaMemcpyHostToDevice, s) != cudaSuccess)
    return ADAMW4_ECUDA;
  StepArgs a = make_args(*cfg, lr, t);
  a.status = status;
  a.fault_stall = g_noalloc_fault_stall.exchange(0);
  StateArena st;
  st.mcodes = state->mcodes;
  st.vcodes = state->vcodes;
  st.mscale = state->mscale;
  st.vscale = state->vscale;
  st.fm = state->m32;
  st.fv = state->v32;
  st.nblocks4 = blocks4;
  st.n32 = elems32;
  st.vs_minus_ms = st.vscale - st.mscale;
  const int64_t need = (unit + kTileUnits - 1) / kTileUnits;
  launch_vcode(cfg->vcode, bf16w, (int)std::min<int64_t>(nd.grid[cfg->vcode][bf16w], need), s,
               table, 0, unit, a, st);
  return cudaGetLastError() == cudaSuccess ? ADAMW4_OK : ADAMW4_ECUDA;
}

extern "C" int adamw4_noalloc_sync(int device, void* cuda_stream) {
  if (device < 0 || device >= kNoAllocMaxDevices) return ADAMW4_EINVAL;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_dev[device].ready) return ADAMW4_EINVAL;
  DeviceGuard dg(device);
  if (!dg.ok) return ADAMW4_ECUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return ADAMW4_ECUDA;
  uint32_t status = 0;
  if (cudaMemcpyFromSymbol(&status, g_noalloc_scratch, sizeof status, 0,
                           cudaMemcpyDeviceToHost) != cudaSuccess)
    return ADAMW4_ECUDA;
  if (status == 0) return ADAMW4_OK;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_noalloc_scratch, &zero, sizeof zero, 0, cudaMemcpyHostToDevice) !=
      cudaSuccess)
    return ADAMW4_ECUDA;
  if (status & 1u) return ADAMW4_ETIMEOUT;
  if (status & 2u) return ADAMW4_ECHECK;
  return ADAMW4_ENONFINITE;
}
