// Host side of the S²-Attn C ABI: argument validation, TMA tensor maps, kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <utility>
#include <vector>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/s2attn.h"
#include "s2_bwd_dkdv.cuh"
#include "s2_bwd_dq.cuh"
#include "s2_bwd_dq_ds.cuh"
#include "s2_bwd_pre.cuh"
#include "s2_rope.cuh"
#include "s2_fwd.cuh"
#include "s2_fwd_sched.h"

namespace {

__device__ unsigned int g_err_word;   // first pipeline-wait failure since the last read

constexpr int kAbiVersion = 5;
constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 1000000000ull;

std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};
thread_local char g_last_error[256] = "";

s2attn_status cuda_fail(cudaError_t e, const char* what) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
  return S2ATTN_ERR_CUDA;
}

struct DeviceState {
  std::once_flag once;
  cudaError_t init_err = cudaSuccess;
  unsigned int* err_word = nullptr;
  int num_sms = 0;
};
DeviceState g_dev[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

template <int D, bool kFront>
cudaError_t set_smem_attrs_variant() {
  cudaError_t e;
  e = cudaFuncSetAttribute(s2::s2_fwd_kernel<D, kFront, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, s2::FwdLayout<D>::kLaunchBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(s2::s2_fwd_kernel<D, kFront, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, s2::FwdLayout<D>::kLaunchBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(s2::s2_bwd_dkdv_kernel<D, kFront>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, s2::DkdvLayout<D>::kLaunchBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(s2::s2_bwd_dq_kernel<D, kFront>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, s2::DqLayout<D>::kLaunchBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(s2::s2_bwd_dq_ds_kernel<D, kFront>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              s2::DqDsLayout<D>::kLaunchBytes);
}
// Every kernel exists twice: with the plain-roll index code only, and with the Variant 3
// reordering compiled in (S2ATTN_FLAG_WRAP_FRONT_FIRST), so the common case pays nothing
// for the general remap.
template <int D>
cudaError_t set_smem_attrs() {
  const cudaError_t e = set_smem_attrs_variant<D, false>();
  return e != cudaSuccess ? e : set_smem_attrs_variant<D, true>();
}

// Per-device one-time set-up (with that device current): the device address of the error
// word, and the kernels' shared-memory limits.
s2attn_status device_state(unsigned int** err_word, int* num_sms = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    std::snprintf(g_last_error, sizeof(g_last_error), "device ordinal %d out of range", dev);
    return S2ATTN_ERR_CUDA;
  }
  DeviceState& s = g_dev[dev];
  std::call_once(s.once, [&] {
    void* p = nullptr;
    s.init_err = cudaGetSymbolAddress(&p, g_err_word);
    if (s.init_err == cudaSuccess) s.init_err = cudaMemset(p, 0, sizeof(unsigned int));
    if (s.init_err == cudaSuccess) s.init_err = set_smem_attrs<64>();
    if (s.init_err == cudaSuccess) s.init_err = set_smem_attrs<128>();
    if (s.init_err == cudaSuccess)
      s.init_err = cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev);
    s.err_word = static_cast<unsigned int*>(p);
  });
  if (s.init_err != cudaSuccess) return cuda_fail(s.init_err, "device set-up");
  *err_word = s.err_word;
  if (num_sms) *num_sms = s.num_sms;
  return S2ATTN_OK;
}

s2attn_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
    return S2ATTN_ERR_CUDA;
  }
  return S2ATTN_OK;
}

// Tensor map over a bf16 [B, N, H, d] tensor: dims (d, H, N, B), box (64, 1, rows, 1),
// 128-byte swizzle, zero fill out of bounds.
s2attn_status encode_map(CUtensorMap* m, const void* base, int B, int H, int N, int d,
                         int box_rows, long long sb, long long st) {
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)st * 2, (cuuint64_t)sb * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return S2ATTN_ERR_CUDA;
  }
  return S2ATTN_OK;
}

struct MapPair {
  CUtensorMap m128, m8;
};
s2attn_status encode_pair(MapPair& mp, const void* base, int B, int H, int N, int d, long long sb,
                          long long st) {
  s2attn_status s = encode_map(&mp.m128, base, B, H, N, d, s2::kTileRows, sb, st);
  if (s != S2ATTN_OK) return s;
  return encode_map(&mp.m8, base, B, H, N, d, 8, sb, st);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace layout: D [B, Hq, N] fp32 | LSE2 [B, Hq, N] fp32 | scheduling words | dS tiles.
// Each array is rounded up to 256 bytes; the scheduling words hold the work counters of the
// persistent gradient kernels ({next, done} for dK/dV, then for dQ).
constexpr size_t kSchedBytes = 256;
constexpr int kSchedWords = static_cast<int>(kSchedBytes / 4);
size_t ws_half(int B, int Hq, int N) {
  const size_t bytes = static_cast<size_t>(B) * Hq * N * sizeof(float);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

// Element strides of each [B, N, H, d] tensor: X[b, t, h, c] is at X + b sb + t st + h d + c
// (the (H, d) block of a token is contiguous). Contiguous tensors have st = H d, sb = N st.
enum TensorId { T_Q = 0, T_K, T_V, T_O, T_DO, T_DQ, T_DK, T_DV, T_COUNT };

struct Shape {
  int B, Hq, Hkv, N, d, G, shb, shift;
  int wrap;   // the shifted heads' wrap split (Variant 2), or s2::kNoWrapSplit
  int front;  // Variant 3: the shifted heads' last group lists the wrapped tokens first
  long long sb[T_COUNT], st[T_COUNT];
  int heads(int t) const { return (t == T_K || t == T_V || t == T_DK || t == T_DV) ? Hkv : Hq; }
  void set_contiguous() {
    for (int t = 0; t < T_COUNT; ++t) {
      st[t] = static_cast<long long>(heads(t)) * d;
      sb[t] = st[t] * N;
    }
  }
};

// dS hand-off (backward without recomputation in the dQ pass): the slot layout, and the bytes
// one kv head (all its query heads, all batches) needs. The dS tiles follow D and LSE2 in the
// workspace.
size_t ws_min_bytes(int B, int Hq, int N) { return 2 * ws_half(B, Hq, N) + kSchedBytes; }
unsigned int* ws_sched(const void* workspace, const Shape& sh) {
  return reinterpret_cast<unsigned int*>(const_cast<char*>(static_cast<const char*>(workspace)) +
                                         2 * ws_half(sh.B, sh.Hq, sh.N));
}

s2::DsSlots ds_layout(const Shape& sh) {
  return s2::ds_slots(sh.N, sh.G, sh.shb < sh.Hq, sh.shift, sh.wrap, sh.front);
}
size_t ds_bytes_per_kv_head(const Shape& sh) {
  const s2::DsSlots sl = ds_layout(sh);
  return static_cast<size_t>(sh.B) * (sh.Hq / sh.Hkv) * static_cast<size_t>(sl.per_head) *
         s2::kDsTileBytes;
}
// kv heads per pass that a workspace of `bytes` allows (0: too small, recompute dQ instead).
int ds_heads_per_pass(const Shape& sh, size_t bytes) {
  const size_t base = ws_min_bytes(sh.B, sh.Hq, sh.N);
  if (bytes <= base) return 0;
  const size_t per = ds_bytes_per_kv_head(sh);
  const size_t k = (bytes - base) / per;
  return k >= static_cast<size_t>(sh.Hkv) ? sh.Hkv : static_cast<int>(k);
}

// Validation shared by every attention entry point (see s2attn.h, "Errors").
s2attn_status check_shape(int B, int Hq, int Hkv, int N, int d, int G, float scale,
                          int shift_head_begin, long long shift, Shape& out, int flags = 0) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0 || G <= 0) return S2ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return S2ATTN_ERR_INVALID_ARG;
  // G must divide N unless the caller asks for a shorter last group
  if (N % G != 0 && !(flags & S2ATTN_FLAG_PARTIAL_LAST_GROUP)) return S2ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return S2ATTN_ERR_INVALID_ARG;
  if (shift_head_begin < 0 || shift_head_begin > Hq) return S2ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return S2ATTN_ERR_UNSUPPORTED;
  if (N >= (1 << 30)) return S2ATTN_ERR_UNSUPPORTED;
  // Any G and roll: tile rows that the 8-row TMA boxes cannot move (a run of the remap that
  // starts or ends inside an 8-row atom) are loaded with plain loads by the producer warps.
  long long s = shift % N;
  if (s < 0) s += N;
  if (shift_head_begin == Hq) s = 0;   // no head is rolled: the roll amount is irrelevant
  const long long rows = static_cast<long long>(B) * (Hq > Hkv ? Hq : Hkv) * ((N + 127) / 128);
  if (rows >= (1ll << 31)) return S2ATTN_ERR_UNSUPPORTED;
  constexpr int kVariants = S2ATTN_FLAG_WRAP_OWN_GROUP | S2ATTN_FLAG_WRAP_FRONT_FIRST;
  if (flags & ~(kVariants | S2ATTN_FLAG_PARTIAL_LAST_GROUP)) return S2ATTN_ERR_INVALID_ARG;
  if ((flags & kVariants) && N % G != 0) return S2ATTN_ERR_INVALID_ARG;   // defined for G | N
  if ((flags & kVariants) == kVariants) return S2ATTN_ERR_INVALID_ARG;   // alternatives
  // the wrap group exists when some head is rolled by 0 < shift < G
  if ((flags & kVariants) && (shift_head_begin >= Hq || s <= 0 || s >= G))
    return S2ATTN_ERR_INVALID_ARG;
  const int wrap = (flags & S2ATTN_FLAG_WRAP_OWN_GROUP) ? N - static_cast<int>(s) : s2::kNoWrapSplit;
  const int front = (flags & S2ATTN_FLAG_WRAP_FRONT_FIRST) ? 1 : 0;
  out = Shape{B, Hq, Hkv, N, d, G, shift_head_begin, static_cast<int>(s), wrap, front, {}, {}};
  out.set_contiguous();
  return S2ATTN_OK;
}

// The forward's per-CTA unit lists (s2::FwdSchedule), built by s2::fwd_unit_lists; round robin
// (count = 0) when the lists would not fit the launch.
void fwd_schedule(const Shape& sh, int grid, s2::FwdSchedule& out) {
  out.count = 0;
  const long long n_units = static_cast<long long>(sh.B) * sh.Hq * s2::query_pairs_per_head(sh.N);
  if (n_units > s2::kFwdSchedMaxUnits || grid > s2::kFwdSchedMaxCtas) return;
  std::vector<int> start, unit;
  if (!s2::fwd_unit_lists(sh.B, sh.Hq, sh.N, sh.G, sh.shb, sh.wrap, grid, start, unit)) return;
  for (int c = 0; c <= grid; ++c) out.start[c] = static_cast<unsigned short>(start[c]);
  for (size_t i = 0; i < unit.size(); ++i) out.unit[i] = static_cast<unsigned short>(unit[i]);
  out.count = static_cast<int>(n_units);
}

// Recently used schedules (the same shapes recur call after call).
struct FwdScheduleCache {
  std::mutex mu;
  struct Entry {
    long long key[9];
    s2::FwdSchedule sched;
  };
  std::vector<Entry> entries;   // most recent last, at most 4
};
FwdScheduleCache g_fwd_sched;

void fwd_schedule_cached(const Shape& sh, int grid, s2::FwdSchedule& out) {
  const long long key[9] = {sh.B, sh.Hq, sh.N, sh.G, sh.shb, sh.shift, sh.wrap, sh.front, grid};
  std::lock_guard<std::mutex> lock(g_fwd_sched.mu);
  auto& es = g_fwd_sched.entries;
  for (size_t i = 0; i < es.size(); ++i)
    if (std::equal(key, key + 9, es[i].key)) {
      out = es[i].sched;
      return;
    }
  fwd_schedule(sh, grid, out);
  if (es.size() == 4) es.erase(es.begin());
  es.emplace_back();
  std::copy(key, key + 9, es.back().key);
  es.back().sched = out;
}

// Fused RoPE of the queries (s2attn_fwd_rope_q): where the rotated queries go and the rotation.
struct RopeArgs {
  void* q_rot = nullptr;
  float log2_base = 0.f, pi_scale = 0.f;
};

template <int D>
s2attn_status launch_fwd(const Shape& sh, const void* q, const void* k, const void* v, void* o,
                         float* lse, float scale, cudaStream_t stream, unsigned int* err,
                         int num_sms, const RopeArgs& rope = RopeArgs{}) {
  MapPair mq, mk, mv;
  s2attn_status s;
  if ((s = encode_pair(mq, q, sh.B, sh.Hq, sh.N, D, sh.sb[T_Q], sh.st[T_Q])) != S2ATTN_OK) return s;
  if ((s = encode_pair(mk, k, sh.B, sh.Hkv, sh.N, D, sh.sb[T_K], sh.st[T_K])) != S2ATTN_OK) return s;
  if ((s = encode_pair(mv, v, sh.B, sh.Hkv, sh.N, D, sh.sb[T_V], sh.st[T_V])) != S2ATTN_OK) return s;
  CUtensorMap mo8;   // O, 8-row boxes: the epilogue's bulk stores
  if ((s = encode_map(&mo8, o, sh.B, sh.Hq, sh.N, D, 8, sh.sb[T_O], sh.st[T_O])) != S2ATTN_OK) return s;
  MapPair mqr = mq;   // the rotated queries (contiguous), stored by the fused RoPE
  if (rope.q_rot) {
    const long long st = static_cast<long long>(sh.Hq) * D;
    if ((s = encode_pair(mqr, rope.q_rot, sh.B, sh.Hq, sh.N, D, st * sh.N, st)) != S2ATTN_OK) return s;
  }
  s2::FwdParams p{};
  p.q = s2::TensorRef{static_cast<const __nv_bfloat16*>(q), sh.sb[T_Q], sh.st[T_Q]};
  p.k = s2::TensorRef{static_cast<const __nv_bfloat16*>(k), sh.sb[T_K], sh.st[T_K]};
  p.v = s2::TensorRef{static_cast<const __nv_bfloat16*>(v), sh.sb[T_V], sh.st[T_V]};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_sb = sh.sb[T_O];
  p.o_st = sh.st[T_O];
  p.lse = lse;
  p.B = sh.B; p.Hq = sh.Hq; p.Hkv = sh.Hkv; p.N = sh.N; p.G = sh.G;
  p.shift_head_begin = sh.shb; p.shift = sh.shift;
  p.wrap = sh.wrap;
  p.front = sh.front;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err;
  p.timeout_ns = g_timeout_ns.load();
  const unsigned units = static_cast<unsigned>(sh.B) * sh.Hq * s2::query_pairs_per_head(sh.N);
  const unsigned grid = units < static_cast<unsigned>(num_sms) ? units : static_cast<unsigned>(num_sms);
  p.q_rot = static_cast<__nv_bfloat16*>(rope.q_rot);
  p.rope_log2_base = rope.log2_base;
  p.rope_pi_scale = rope.pi_scale;
  static thread_local s2::FwdSchedule sched;
  fwd_schedule_cached(sh, static_cast<int>(grid), sched);
  constexpr uint32_t kSmem = s2::FwdLayout<D>::kLaunchBytes;
  constexpr int kT = s2::FwdLayout<D>::kThreads, kTR = s2::FwdLayout<D>::kRopeThreads;
  if (rope.q_rot && sh.front)
    s2::s2_fwd_kernel<D, true, true><<<grid, kTR, kSmem, stream>>>(mq.m128, mq.m8, mk.m128, mk.m8,
                                                                   mv.m128, mv.m8, mo8, mqr.m128, mqr.m8, p, sched);
  else if (rope.q_rot)
    s2::s2_fwd_kernel<D, false, true><<<grid, kTR, kSmem, stream>>>(mq.m128, mq.m8, mk.m128, mk.m8,
                                                                    mv.m128, mv.m8, mo8, mqr.m128, mqr.m8, p, sched);
  else if (sh.front)
    s2::s2_fwd_kernel<D, true, false><<<grid, kT, kSmem, stream>>>(mq.m128, mq.m8, mk.m128, mk.m8,
                                                                   mv.m128, mv.m8, mo8, mqr.m128, mqr.m8, p, sched);
  else
    s2::s2_fwd_kernel<D, false, false><<<grid, kT, kSmem, stream>>>(mq.m128, mq.m8, mk.m128, mk.m8,
                                                                    mv.m128, mv.m8, mo8, mqr.m128, mqr.m8, p, sched);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? S2ATTN_OK : cuda_fail(e, "s2_fwd_kernel launch");
}

s2::BwdParams bwd_params(const Shape& sh, float scale, const void* workspace, void* dq, void* dk,
                         void* dv, unsigned int* err) {
  s2::BwdParams p{};
  const size_t half = ws_half(sh.B, sh.Hq, sh.N);
  p.dvec = static_cast<const float*>(workspace);
  p.lse2 = reinterpret_cast<const float*>(static_cast<const char*>(workspace) + half);
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.B = sh.B; p.Hq = sh.Hq; p.Hkv = sh.Hkv; p.N = sh.N; p.G = sh.G;
  p.shift_head_begin = sh.shb; p.shift = sh.shift;
  p.wrap = sh.wrap;
  p.front = sh.front;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err;
  p.timeout_ns = g_timeout_ns.load();
  p.dq_sb = sh.sb[T_DQ];
  p.dq_st = sh.st[T_DQ];
  p.kvh_begin = 0;
  p.kvh_count = sh.Hkv;
  p.ds = nullptr;
  p.slots = s2::DsSlots{};
  p.sched = ws_sched(workspace, sh);
  return p;
}

// Point the parameters at the dS region of the workspace for kv heads [kvh_begin, +count).
void set_ds_pass(s2::BwdParams& p, const Shape& sh, const void* workspace, int kvh_begin,
                 int kvh_count) {
  p.kvh_begin = kvh_begin;
  p.kvh_count = kvh_count;
  p.slots = ds_layout(sh);
  p.ds = reinterpret_cast<__nv_bfloat16*>(const_cast<char*>(static_cast<const char*>(workspace)) +
                                          ws_min_bytes(sh.B, sh.Hq, sh.N));
}

template <int D>
s2attn_status launch_pre(const Shape& sh, const void* o, const float* lse, const void* dO,
                         void* workspace, cudaStream_t stream) {
  const size_t half = ws_half(sh.B, sh.Hq, sh.N);
  float* dvec = static_cast<float*>(workspace);
  float* lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + half);
  const unsigned grid = static_cast<unsigned>(sh.B) * ((sh.N + s2::kPreTokens - 1) / s2::kPreTokens);
  s2::s2_bwd_pre_kernel<D><<<grid, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, dvec,
      lse2, ws_sched(workspace, sh), kSchedWords, sh.Hq, sh.N, sh.sb[T_O], sh.st[T_O],
      sh.sb[T_DO], sh.st[T_DO]);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? S2ATTN_OK : cuda_fail(e, "s2_bwd_pre_kernel launch");
}

template <int D, bool kDkdv>
s2attn_status launch_grad(const Shape& sh, const void* q, const void* k, const void* v,
                          const void* dO, void* dq, void* dk, void* dv, float scale,
                          const void* workspace, cudaStream_t stream, unsigned int* err,
                          int num_sms, int ds_kvh_begin = -1, int ds_kvh_count = 0) {
  MapPair mq, mk, mv, mo;
  s2attn_status s;
  if ((s = encode_pair(mq, q, sh.B, sh.Hq, sh.N, D, sh.sb[T_Q], sh.st[T_Q])) != S2ATTN_OK) return s;
  if ((s = encode_pair(mk, k, sh.B, sh.Hkv, sh.N, D, sh.sb[T_K], sh.st[T_K])) != S2ATTN_OK) return s;
  if ((s = encode_pair(mv, v, sh.B, sh.Hkv, sh.N, D, sh.sb[T_V], sh.st[T_V])) != S2ATTN_OK) return s;
  if ((s = encode_pair(mo, dO, sh.B, sh.Hq, sh.N, D, sh.sb[T_DO], sh.st[T_DO])) != S2ATTN_OK) return s;
  s2::BwdParams p = bwd_params(sh, scale, workspace, dq, dk, dv, err);
  p.q = s2::TensorRef{static_cast<const __nv_bfloat16*>(q), sh.sb[T_Q], sh.st[T_Q]};
  p.k = s2::TensorRef{static_cast<const __nv_bfloat16*>(k), sh.sb[T_K], sh.st[T_K]};
  p.v = s2::TensorRef{static_cast<const __nv_bfloat16*>(v), sh.sb[T_V], sh.st[T_V]};
  p.dO = s2::TensorRef{static_cast<const __nv_bfloat16*>(dO), sh.sb[T_DO], sh.st[T_DO]};
  if (ds_kvh_begin >= 0) set_ds_pass(p, sh, workspace, ds_kvh_begin, ds_kvh_count);
  const unsigned tiles = (sh.N + 127) / 128;
  if (kDkdv) {
    MapPair mdk, mdv;
    if ((s = encode_pair(mdk, dk, sh.B, sh.Hkv, sh.N, D, sh.sb[T_DK], sh.st[T_DK])) != S2ATTN_OK)
      return s;
    if ((s = encode_pair(mdv, dv, sh.B, sh.Hkv, sh.N, D, sh.sb[T_DV], sh.st[T_DV])) != S2ATTN_OK)
      return s;
    const unsigned units = static_cast<unsigned>(sh.B) * p.kvh_count * tiles;
    const unsigned grid = units < static_cast<unsigned>(num_sms) ? units : static_cast<unsigned>(num_sms);
    if (sh.front)
      s2::s2_bwd_dkdv_kernel<D, true><<<grid, s2::DkdvLayout<D>::kThreads,
                                        s2::DkdvLayout<D>::kLaunchBytes, stream>>>(
          mq.m128, mq.m8, mk.m128, mk.m8, mv.m128, mv.m8, mo.m128, mo.m8, mdk.m128, mdv.m128, p);
    else
      s2::s2_bwd_dkdv_kernel<D, false><<<grid, s2::DkdvLayout<D>::kThreads,
                                         s2::DkdvLayout<D>::kLaunchBytes, stream>>>(
          mq.m128, mq.m8, mk.m128, mk.m8, mv.m128, mv.m8, mo.m128, mo.m8, mdk.m128, mdv.m128, p);
  } else {
    const unsigned grid = static_cast<unsigned>(sh.B) * sh.Hq * tiles;
    if (sh.front)
      s2::s2_bwd_dq_kernel<D, true><<<grid, s2::DqLayout<D>::kThreads, s2::DqLayout<D>::kLaunchBytes,
                                      stream>>>(mq.m128, mq.m8, mk.m128, mk.m8, mv.m128, mv.m8,
                                                mo.m128, mo.m8, p);
    else
      s2::s2_bwd_dq_kernel<D, false><<<grid, s2::DqLayout<D>::kThreads, s2::DqLayout<D>::kLaunchBytes,
                                       stream>>>(mq.m128, mq.m8, mk.m128, mk.m8, mv.m128, mv.m8,
                                                 mo.m128, mo.m8, p);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? S2ATTN_OK
                          : cuda_fail(e, kDkdv ? "s2_bwd_dkdv_kernel launch" : "s2_bwd_dq_kernel launch");
}

template <int D>
s2attn_status launch_dq_ds(const Shape& sh, const void* k, void* dq, float scale,
                           const void* workspace, int kvh_begin, int kvh_count,
                           cudaStream_t stream, unsigned int* err, int num_sms) {
  MapPair mk;
  s2attn_status s;
  if ((s = encode_pair(mk, k, sh.B, sh.Hkv, sh.N, D, sh.sb[T_K], sh.st[T_K])) != S2ATTN_OK) return s;
  CUtensorMap mdq8;   // dQ, 8-row boxes: the epilogue's bulk stores
  if ((s = encode_map(&mdq8, dq, sh.B, sh.Hq, sh.N, D, 8, sh.sb[T_DQ], sh.st[T_DQ])) != S2ATTN_OK)
    return s;
  s2::BwdParams p = bwd_params(sh, scale, workspace, dq, nullptr, nullptr, err);
  set_ds_pass(p, sh, workspace, kvh_begin, kvh_count);
  p.sched = ws_sched(workspace, sh) + 2;
  const unsigned units = static_cast<unsigned>(sh.B) * kvh_count * (sh.Hq / sh.Hkv) *
                         ((sh.N + 127) / 128);
  const unsigned grid = units < static_cast<unsigned>(num_sms) ? units : static_cast<unsigned>(num_sms);
  if (sh.front)
    s2::s2_bwd_dq_ds_kernel<D, true><<<grid, s2::DqDsLayout<D>::kThreads,
                                       s2::DqDsLayout<D>::kLaunchBytes, stream>>>(mk.m128, mk.m8, mdq8, p);
  else
    s2::s2_bwd_dq_ds_kernel<D, false><<<grid, s2::DqDsLayout<D>::kThreads,
                                        s2::DqDsLayout<D>::kLaunchBytes, stream>>>(mk.m128, mk.m8, mdq8, p);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? S2ATTN_OK : cuda_fail(e, "s2_bwd_dq_ds_kernel launch");
}

s2attn_status check_workspace(const Shape& sh, const void* ws, size_t bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return S2ATTN_ERR_INVALID_ARG;
  if (bytes < ws_min_bytes(sh.B, sh.Hq, sh.N)) return S2ATTN_ERR_INVALID_ARG;
  return S2ATTN_OK;
}

s2attn_status dkdv_impl(const Shape& sh, const void* q, const void* k, const void* v,
                        const void* dO, void* dk, void* dv, float scale, const void* ws,
                        cudaStream_t stream, unsigned int* err, int num_sms) {
  return sh.d == 64 ? launch_grad<64, true>(sh, q, k, v, dO, nullptr, dk, dv, scale, ws, stream, err, num_sms)
                    : launch_grad<128, true>(sh, q, k, v, dO, nullptr, dk, dv, scale, ws, stream, err, num_sms);
}
s2attn_status dq_impl(const Shape& sh, const void* q, const void* k, const void* v,
                      const void* dO, void* dq, float scale, const void* ws, cudaStream_t stream,
                      unsigned int* err) {
  return sh.d == 64 ? launch_grad<64, false>(sh, q, k, v, dO, dq, nullptr, nullptr, scale, ws, stream, err, 0)
                    : launch_grad<128, false>(sh, q, k, v, dO, dq, nullptr, nullptr, scale, ws, stream, err, 0);
}
s2attn_status dkdv_ds_impl(const Shape& sh, const void* q, const void* k, const void* v,
                           const void* dO, void* dk, void* dv, float scale, const void* ws,
                           int kvh_begin, int kvh_count, cudaStream_t stream, unsigned int* err,
                           int num_sms) {
  return sh.d == 64
             ? launch_grad<64, true>(sh, q, k, v, dO, nullptr, dk, dv, scale, ws, stream, err,
                                     num_sms, kvh_begin, kvh_count)
             : launch_grad<128, true>(sh, q, k, v, dO, nullptr, dk, dv, scale, ws, stream, err,
                                      num_sms, kvh_begin, kvh_count);
}
s2attn_status dq_ds_impl(const Shape& sh, const void* k, void* dq, float scale, const void* ws,
                         int kvh_begin, int kvh_count, cudaStream_t stream, unsigned int* err,
                         int num_sms) {
  return sh.d == 64 ? launch_dq_ds<64>(sh, k, dq, scale, ws, kvh_begin, kvh_count, stream, err, num_sms)
                    : launch_dq_ds<128>(sh, k, dq, scale, ws, kvh_begin, kvh_count, stream, err, num_sms);
}
s2attn_status pre_impl(const Shape& sh, const void* o, const float* lse, const void* dO, void* ws,
                       cudaStream_t stream) {
  return sh.d == 64 ? launch_pre<64>(sh, o, lse, dO, ws, stream)
                    : launch_pre<128>(sh, o, lse, dO, ws, stream);
}

// Caller-given strides for tensors ids[0..n): strides[2i] = batch, strides[2i+1] = token (in
// elements). Each must be a multiple of 8 (16 bytes, the TMA rule), the token stride must span
// the token's (H, d) block, and batches must not overlap.
s2attn_status apply_strides(Shape& sh, const long long* strides, const int* ids, int n) {
  if (!strides) return S2ATTN_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const long long sb = strides[2 * i], st = strides[2 * i + 1];
    const int t = ids[i];
    if (sb < 0 || st < static_cast<long long>(sh.heads(t)) * sh.d || sb % 8 != 0 || st % 8 != 0)
      return S2ATTN_ERR_INVALID_ARG;
    if (sh.B > 1 && sb < st * sh.N) return S2ATTN_ERR_INVALID_ARG;
    if (st >= (1ll << 37) || sb >= (1ll << 38)) return S2ATTN_ERR_UNSUPPORTED;   // TMA stride range
    sh.sb[t] = sb;
    sh.st[t] = st;
  }
  return S2ATTN_OK;
}

// Self-test kernel: a bounded wait on a barrier that nothing arrives on.
__global__ void selftest_wait_kernel(unsigned int* err, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t barrier;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    s2::mbar_init(s2::smem_u32(&barrier), 1);
    s2::fence_barrier_init();
  }
  __syncthreads();
  const s2::WaitCtx ctx{&abort_flag, err, timeout_ns, s2::KID_SELFTEST};
  s2::wait_bar(s2::smem_u32(&barrier), 0, ctx, 1);
  __syncthreads();
}

}  // namespace

extern "C" {

int s2attn_abi_version(void) { return kAbiVersion; }

const char* s2attn_status_string(int status) {
  switch (status) {
    case S2ATTN_OK: return "ok";
    case S2ATTN_ERR_INVALID_ARG: return "invalid argument";
    case S2ATTN_ERR_UNSUPPORTED: return "unsupported shape";
    case S2ATTN_ERR_CUDA: return "CUDA error";
    case S2ATTN_ERR_TIMEOUT: return "kernel pipeline wait timed out";
    default: return "unknown status";
  }
}

const char* s2attn_last_error(void) { return g_last_error; }

void s2attn_set_wait_timeout_ns(unsigned long long ns) {
  g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : ns);
}

s2attn_status s2attn_fwd_general(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int B, int Hq, int Hkv, int N, int d, int G, float scale,
                                 int shift_head_begin, int shift, int flags,
                                 const long long* strides, void* stream) {
  if (!q || !k || !v || !o || !lse) return S2ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return S2ATTN_ERR_INVALID_ARG;
  Shape sh;
  s2attn_status s = check_shape(B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift, sh, flags);
  if (s != S2ATTN_OK) return s;
  if (strides) {
    static const int ids[4] = {T_Q, T_K, T_V, T_O};
    if ((s = apply_strides(sh, strides, ids, 4)) != S2ATTN_OK) return s;
  }
  if ((s = get_encoder()) != S2ATTN_OK) return s;
  unsigned int* err = nullptr;
  int num_sms = 0;
  if ((s = device_state(&err, &num_sms)) != S2ATTN_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_fwd<64>(sh, q, k, v, o, lse, scale, st, err, num_sms)
                 : launch_fwd<128>(sh, q, k, v, o, lse, scale, st, err, num_sms);
}

s2attn_status s2attn_fwd_rope_q(const void* q, const void* k, const void* v, void* o, float* lse,
                                void* q_rot, int B, int Hq, int Hkv, int N, int d, int G,
                                float scale, int shift_head_begin, int shift, int flags,
                                float base, float pi_scale, void* stream) {
  if (!q || !k || !v || !o || !lse || !q_rot) return S2ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(q_rot))
    return S2ATTN_ERR_INVALID_ARG;
  if (!(base > 1.f) || !std::isfinite(base) || !(pi_scale > 0.f) || !std::isfinite(pi_scale))
    return S2ATTN_ERR_INVALID_ARG;
  Shape sh;
  s2attn_status s = check_shape(B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift, sh, flags);
  if (s != S2ATTN_OK) return s;
  if (N >= (1 << 24)) return S2ATTN_ERR_UNSUPPORTED;   // positions exact in fp32, as s2attn_rope_pi
  if ((s = get_encoder()) != S2ATTN_OK) return s;
  unsigned int* err = nullptr;
  int num_sms = 0;
  if ((s = device_state(&err, &num_sms)) != S2ATTN_OK) return s;
  RopeArgs rope;
  rope.q_rot = q_rot;
  rope.log2_base = std::log2(base);
  rope.pi_scale = pi_scale;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_fwd<64>(sh, q, k, v, o, lse, scale, st, err, num_sms, rope)
                 : launch_fwd<128>(sh, q, k, v, o, lse, scale, st, err, num_sms, rope);
}

s2attn_status s2attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int Hq, int Hkv, int N, int d, int G, float scale,
                            int shift_head_begin, int shift, void* stream) {
  // null strides: contiguous tensors
  return s2attn_fwd_general(q, k, v, o, lse, B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift,
                            0, nullptr, stream);
}

s2attn_status s2attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int Hq, int Hkv, int N, int d, int G, float scale,
                         void* stream) {
  if (Hq <= 0 || Hq % 2 != 0) return S2ATTN_ERR_INVALID_ARG;
  return s2attn_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, N, d, G, scale, Hq / 2, G / 2, stream);
}

size_t s2attn_bwd_workspace_size(int B, int Hq, int N) {
  if (B <= 0 || Hq <= 0 || N <= 0) return 0;
  return ws_min_bytes(B, Hq, N);
}

size_t s2attn_bwd_workspace_size_general(int B, int Hq, int Hkv, int N, int d, int G,
                                         int shift_head_begin, int shift, int flags,
                                         size_t cap_bytes) {
  Shape sh;
  if (check_shape(B, Hq, Hkv, N, d, G, 1.0f, shift_head_begin, shift, sh, flags) != S2ATTN_OK)
    return 0;
  const size_t base = ws_min_bytes(B, Hq, N);
  const size_t per = ds_bytes_per_kv_head(sh);
  size_t k = static_cast<size_t>(Hkv);
  if (cap_bytes != 0) {
    const size_t fit = cap_bytes > base ? (cap_bytes - base) / per : 0;
    k = fit < k ? fit : k;
    if (k == 0) k = 1;
  }
  return base + k * per;
}

size_t s2attn_bwd_workspace_size_ex(int B, int Hq, int Hkv, int N, int d, int G,
                                    int shift_head_begin, int shift, size_t cap_bytes) {
  return s2attn_bwd_workspace_size_general(B, Hq, Hkv, N, d, G, shift_head_begin, shift, 0,
                                           cap_bytes);
}

s2attn_status s2attn_bwd_preprocess(const void* o, const float* lse, const void* dO, int B,
                                    int Hq, int N, int d, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (!o || !lse || !dO || !aligned16(o) || !aligned16(dO) || !aligned16(lse))
    return S2ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || N <= 0 || d <= 0) return S2ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return S2ATTN_ERR_UNSUPPORTED;
  if (N >= (1 << 30) || static_cast<long long>(B) * Hq * ((N + 127) / 128) >= (1ll << 31))
    return S2ATTN_ERR_UNSUPPORTED;
  Shape sh{B, Hq, Hq, N, d, N, Hq, 0, s2::kNoWrapSplit, 0, {}, {}};
  sh.set_contiguous();
  s2attn_status s = check_workspace(sh, workspace, workspace_bytes);
  if (s != S2ATTN_OK) return s;
  return pre_impl(sh, o, lse, dO, workspace, static_cast<cudaStream_t>(stream));
}

s2attn_status s2attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO,
                              void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int G,
                              float scale, int shift_head_begin, int shift,
                              const void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !dO || !dk || !dv) return S2ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk) ||
      !aligned16(dv))
    return S2ATTN_ERR_INVALID_ARG;
  Shape sh;
  s2attn_status s = check_shape(B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift, sh);
  if (s != S2ATTN_OK) return s;
  if ((s = check_workspace(sh, workspace, workspace_bytes)) != S2ATTN_OK) return s;
  if ((s = get_encoder()) != S2ATTN_OK) return s;
  unsigned int* err = nullptr;
  int num_sms = 0;
  if ((s = device_state(&err, &num_sms)) != S2ATTN_OK) return s;
  return dkdv_impl(sh, q, k, v, dO, dk, dv, scale, workspace, static_cast<cudaStream_t>(stream), err,
                   num_sms);
}

s2attn_status s2attn_bwd_dq(const void* q, const void* k, const void* v, const void* dO,
                            void* dq, int B, int Hq, int Hkv, int N, int d, int G, float scale,
                            int shift_head_begin, int shift, const void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !dO || !dq) return S2ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dq))
    return S2ATTN_ERR_INVALID_ARG;
  Shape sh;
  s2attn_status s = check_shape(B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift, sh);
  if (s != S2ATTN_OK) return s;
  if ((s = check_workspace(sh, workspace, workspace_bytes)) != S2ATTN_OK) return s;
  if ((s = get_encoder()) != S2ATTN_OK) return s;
  unsigned int* err = nullptr;
  if ((s = device_state(&err)) != S2ATTN_OK) return s;
  return dq_impl(sh, q, k, v, dO, dq, scale, workspace, static_cast<cudaStream_t>(stream), err);
}

s2attn_status s2attn_bwd_dkdv_ds(const void* q, const void* k, const void* v, const void* dO,
                                 void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int G,
                                 float scale, int shift_head_begin, int shift, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !dO || !dk || !dv) return S2ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk) ||
      !aligned16(dv))
    return S2ATTN_ERR_INVALID_ARG;
  Shape sh;
  s2attn_status s = check_shape(B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift, sh);
  if (s != S2ATTN_OK) return s;
  if ((s = check_workspace(sh, workspace, workspace_bytes)) != S2ATTN_OK) return s;
  if (ds_heads_per_pass(sh, workspace_bytes) < Hkv) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "s2attn_bwd_dkdv_ds: workspace of %zu bytes holds the dS tiles of fewer than "
                  "all %d kv heads", workspace_bytes, Hkv);
    return S2ATTN_ERR_INVALID_ARG;
  }
  if ((s = get_encoder()) != S2ATTN_OK) return s;
  unsigned int* err = nullptr;
  int num_sms = 0;
  if ((s = device_state(&err, &num_sms)) != S2ATTN_OK) return s;
  return dkdv_ds_impl(sh, q, k, v, dO, dk, dv, scale, workspace, 0, Hkv,
                      static_cast<cudaStream_t>(stream), err, num_sms);
}

s2attn_status s2attn_bwd_dq_ds(const void* k, void* dq, int B, int Hq, int Hkv, int N, int d,
                               int G, float scale, int shift_head_begin, int shift,
                               const void* workspace, size_t workspace_bytes, void* stream) {
  if (!k || !dq || !aligned16(k) || !aligned16(dq)) return S2ATTN_ERR_INVALID_ARG;
  Shape sh;
  s2attn_status s = check_shape(B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift, sh);
  if (s != S2ATTN_OK) return s;
  if ((s = check_workspace(sh, workspace, workspace_bytes)) != S2ATTN_OK) return s;
  if (ds_heads_per_pass(sh, workspace_bytes) < Hkv) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "s2attn_bwd_dq_ds: workspace of %zu bytes holds the dS tiles of fewer than "
                  "all %d kv heads", workspace_bytes, Hkv);
    return S2ATTN_ERR_INVALID_ARG;
  }
  if ((s = get_encoder()) != S2ATTN_OK) return s;
  unsigned int* err = nullptr;
  int num_sms = 0;
  if ((s = device_state(&err, &num_sms)) != S2ATTN_OK) return s;
  return dq_ds_impl(sh, k, dq, scale, workspace, 0, Hkv, static_cast<cudaStream_t>(stream), err,
                    num_sms);
}

// Shape, option flags and strides of the phase entry points (strides: the 8 {sb, st} pairs of
// s2attn_bwd_general; the pairs of tensors a phase does not touch are validated all the same).
s2attn_status phase_shape(int B, int Hq, int Hkv, int N, int d, int G, float scale,
                          int shift_head_begin, int shift, int flags, const long long* strides,
                          Shape& sh) {
  s2attn_status s = check_shape(B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift, sh, flags);
  if (s != S2ATTN_OK) return s;
  if (strides) {
    static const int ids[8] = {T_Q, T_K, T_V, T_O, T_DO, T_DQ, T_DK, T_DV};
    if ((s = apply_strides(sh, strides, ids, 8)) != S2ATTN_OK) return s;
  }
  return S2ATTN_OK;
}

s2attn_status s2attn_bwd_dkdv_ds_general(const void* q, const void* k, const void* v,
                                         const void* dO, void* dk, void* dv, int B, int Hq,
                                         int Hkv, int N, int d, int G, float scale,
                                         int shift_head_begin, int shift, int flags,
                                         const long long* strides, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !dO || !dk || !dv) return S2ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk) ||
      !aligned16(dv))
    return S2ATTN_ERR_INVALID_ARG;
  Shape sh;
  s2attn_status s = phase_shape(B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift, flags,
                                strides, sh);
  if (s != S2ATTN_OK) return s;
  if ((s = check_workspace(sh, workspace, workspace_bytes)) != S2ATTN_OK) return s;
  if (ds_heads_per_pass(sh, workspace_bytes) < Hkv) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "s2attn_bwd_dkdv_ds_general: workspace of %zu bytes holds the dS tiles of fewer "
                  "than all %d kv heads", workspace_bytes, Hkv);
    return S2ATTN_ERR_INVALID_ARG;
  }
  if ((s = get_encoder()) != S2ATTN_OK) return s;
  unsigned int* err = nullptr;
  int num_sms = 0;
  if ((s = device_state(&err, &num_sms)) != S2ATTN_OK) return s;
  return dkdv_ds_impl(sh, q, k, v, dO, dk, dv, scale, workspace, 0, Hkv,
                      static_cast<cudaStream_t>(stream), err, num_sms);
}

s2attn_status s2attn_bwd_dq_ds_general(const void* k, void* dq, int B, int Hq, int Hkv, int N,
                                       int d, int G, float scale, int shift_head_begin,
                                       int shift, int flags, const long long* strides,
                                       const void* workspace, size_t workspace_bytes,
                                       void* stream) {
  if (!k || !dq || !aligned16(k) || !aligned16(dq)) return S2ATTN_ERR_INVALID_ARG;
  Shape sh;
  s2attn_status s = phase_shape(B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift, flags,
                                strides, sh);
  if (s != S2ATTN_OK) return s;
  if ((s = check_workspace(sh, workspace, workspace_bytes)) != S2ATTN_OK) return s;
  if (ds_heads_per_pass(sh, workspace_bytes) < Hkv) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "s2attn_bwd_dq_ds_general: workspace of %zu bytes holds the dS tiles of fewer "
                  "than all %d kv heads", workspace_bytes, Hkv);
    return S2ATTN_ERR_INVALID_ARG;
  }
  if ((s = get_encoder()) != S2ATTN_OK) return s;
  unsigned int* err = nullptr;
  int num_sms = 0;
  if ((s = device_state(&err, &num_sms)) != S2ATTN_OK) return s;
  return dq_ds_impl(sh, k, dq, scale, workspace, 0, Hkv, static_cast<cudaStream_t>(stream), err,
                    num_sms);
}

s2attn_status s2attn_bwd_general(const void* q, const void* k, const void* v, const void* o,
                                 const float* lse, const void* dO, void* dq, void* dk, void* dv,
                                 int B, int Hq, int Hkv, int N, int d, int G, float scale,
                                 int shift_head_begin, int shift, int flags,
                                 const long long* strides, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return S2ATTN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, lse, dO, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return S2ATTN_ERR_INVALID_ARG;
  Shape sh;
  s2attn_status s = check_shape(B, Hq, Hkv, N, d, G, scale, shift_head_begin, shift, sh, flags);
  if (s != S2ATTN_OK) return s;
  if (strides) {
    static const int ids[8] = {T_Q, T_K, T_V, T_O, T_DO, T_DQ, T_DK, T_DV};
    if ((s = apply_strides(sh, strides, ids, 8)) != S2ATTN_OK) return s;
  }
  if ((s = check_workspace(sh, workspace, workspace_bytes)) != S2ATTN_OK) return s;
  if ((s = get_encoder()) != S2ATTN_OK) return s;
  unsigned int* err = nullptr;
  int num_sms = 0;
  if ((s = device_state(&err, &num_sms)) != S2ATTN_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = pre_impl(sh, o, lse, dO, workspace, st)) != S2ATTN_OK) return s;
  const int per_pass = ds_heads_per_pass(sh, workspace_bytes);
  if (per_pass == 0) {
    // Workspace too small for one kv head's dS tiles: the dQ kernel recomputes S and dP.
    if ((s = dkdv_impl(sh, q, k, v, dO, dk, dv, scale, workspace, st, err, num_sms)) != S2ATTN_OK)
      return s;
    return dq_impl(sh, q, k, v, dO, dq, scale, workspace, st, err);
  }
  for (int h0 = 0; h0 < sh.Hkv; h0 += per_pass) {
    const int cnt = sh.Hkv - h0 < per_pass ? sh.Hkv - h0 : per_pass;
    if ((s = dkdv_ds_impl(sh, q, k, v, dO, dk, dv, scale, workspace, h0, cnt, st, err, num_sms)) !=
        S2ATTN_OK)
      return s;
    if ((s = dq_ds_impl(sh, k, dq, scale, workspace, h0, cnt, st, err, num_sms)) != S2ATTN_OK)
      return s;
  }
  return S2ATTN_OK;
}

s2attn_status s2attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, void* dq, void* dk, void* dv,
                            int B, int Hq, int Hkv, int N, int d, int G, float scale,
                            int shift_head_begin, int shift, void* workspace,
                            size_t workspace_bytes, void* stream) {
  // null strides: contiguous tensors
  return s2attn_bwd_general(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, N, d, G, scale,
                            shift_head_begin, shift, 0, nullptr, workspace, workspace_bytes, stream);
}

s2attn_status s2attn_bwd(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dO, void* dq, void* dk, void* dv,
                         int B, int Hq, int Hkv, int N, int d, int G, float scale,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (Hq <= 0 || Hq % 2 != 0) return S2ATTN_ERR_INVALID_ARG;
  return s2attn_bwd_ex(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, N, d, G, scale, Hq / 2,
                       G / 2, workspace, workspace_bytes, stream);
}

s2attn_status s2attn_get_device_error(void* stream, unsigned int* code_out) {
  if (code_out) *code_out = 0;
  unsigned int* err = nullptr;
  s2attn_status s = device_state(&err);
  if (s != S2ATTN_OK) return s;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int code = 0;
  e = cudaMemcpy(&code, err, sizeof(code), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the error word");
  if (code != 0) {
    e = cudaMemset(err, 0, sizeof(unsigned int));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  }
  if (code_out) *code_out = code;
  return code != 0 ? S2ATTN_ERR_TIMEOUT : S2ATTN_OK;
}

s2attn_status s2attn_selftest_wait_timeout(unsigned long long timeout_ns, void* stream) {
  unsigned int* err = nullptr;
  s2attn_status s = device_state(&err);
  if (s != S2ATTN_OK) return s;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, timeout_ns);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? S2ATTN_OK : cuda_fail(e, "selftest_wait_kernel launch");
}

s2attn_status s2attn_rope_pi(const void* x, void* y, int B, int N, int H, int d, float base,
                             float pi_scale, int inverse, const long long* strides,
                             void* stream) {
  if (!x || !y || !aligned16(x) || !aligned16(y)) return S2ATTN_ERR_INVALID_ARG;
  if (B <= 0 || N <= 0 || H <= 0 || d <= 0) return S2ATTN_ERR_INVALID_ARG;
  if (!(base > 1.f) || !std::isfinite(base) || !(pi_scale > 0.f) || !std::isfinite(pi_scale))
    return S2ATTN_ERR_INVALID_ARG;
  if (inverse != 0 && inverse != 1) return S2ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return S2ATTN_ERR_UNSUPPORTED;
  if (N >= (1 << 24) || static_cast<long long>(H) * d >= (1ll << 31)) return S2ATTN_ERR_UNSUPPORTED;
  long long st[4] = {static_cast<long long>(N) * H * d, static_cast<long long>(H) * d,
                     static_cast<long long>(N) * H * d, static_cast<long long>(H) * d};
  if (strides) {
    for (int i = 0; i < 2; ++i) {
      const long long sb = strides[2 * i], stt = strides[2 * i + 1];
      if (sb < 0 || stt < static_cast<long long>(H) * d || sb % 8 != 0 || stt % 8 != 0)
        return S2ATTN_ERR_INVALID_ARG;
      if (B > 1 && sb < stt * N) return S2ATTN_ERR_INVALID_ARG;
      st[2 * i] = sb;
      st[2 * i + 1] = stt;
    }
  }
  const long long blocks = static_cast<long long>(B) * ((N + s2::kRopeTokens - 1) / s2::kRopeTokens);
  if (blocks >= (1ll << 31)) return S2ATTN_ERR_UNSUPPORTED;
  const float log2_base = std::log2(base);
  const float sign = inverse ? -1.f : 1.f;
  cudaStream_t sm = static_cast<cudaStream_t>(stream);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* yb = static_cast<__nv_bfloat16*>(y);
  if (d == 64)
    s2::s2_rope_kernel<64><<<static_cast<unsigned>(blocks), s2::kRopeThreads, 0, sm>>>(
        xb, yb, N, H, st[0], st[1], st[2], st[3], log2_base, pi_scale, sign);
  else
    s2::s2_rope_kernel<128><<<static_cast<unsigned>(blocks), s2::kRopeThreads, 0, sm>>>(
        xb, yb, N, H, st[0], st[1], st[2], st[3], log2_base, pi_scale, sign);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? S2ATTN_OK : cuda_fail(e, "s2_rope_kernel launch");
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// Allocation-free backward: the workspace is a static device array of this file.
// ------------------------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocRowBytes = size_t(16) << 20;        // 16 MiB: 2^21 rows of D + LSE2
constexpr size_t kNoAllocScratchBytes = kNoAllocRowBytes + kSchedBytes;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocScratch {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  void* ptr = nullptr;   // device address of g_noalloc_scratch on this device
};
NoAllocScratch g_noalloc[kMaxDevices];

// Device address of the static scratch for the current device. In host code the array's name
// only stands in for the symbol; the address the kernels need comes from the runtime, looked
// up once per device with that device current.
s2attn_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    std::snprintf(g_last_error, sizeof(g_last_error), "device ordinal %d out of range", dev);
    return S2ATTN_ERR_CUDA;
  }
  NoAllocScratch& s = g_noalloc[dev];
  std::call_once(s.once, [&] {
    void* p = nullptr;
    s.err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    s.ptr = p;
  });
  if (s.err != cudaSuccess) return cuda_fail(s.err, "cudaGetSymbolAddress(static scratch)");
  *out = s.ptr;
  return S2ATTN_OK;
}

}  // namespace

extern "C" s2attn_status s2attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                            const void* o, const float* lse, const void* dO,
                                            void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                                            int N, int d, int G, float scale, void* stream) {
  if (B > 0 && Hq > 0 && N > 0 &&
      2 * ws_half(B, Hq, N) > kNoAllocRowBytes) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "s2attn_bwd_noalloc: B*Hq*N = %lld rows need %zu scratch bytes; the static "
                  "scratch holds %zu (at most 2097152 rows)",
                  static_cast<long long>(B) * Hq * N, 2 * ws_half(B, Hq, N), kNoAllocRowBytes);
    return S2ATTN_ERR_UNSUPPORTED;
  }
  if (Hq <= 0 || Hq % 2 != 0) return S2ATTN_ERR_INVALID_ARG;
  void* scratch = nullptr;
  s2attn_status s = noalloc_scratch(&scratch);
  if (s != S2ATTN_OK) return s;
  return s2attn_bwd_ex(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, N, d, G, scale, Hq / 2, G / 2,
                       scratch, kNoAllocScratchBytes, stream);
}
