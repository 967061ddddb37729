// vsa_api.cu -- the C ABI declared in include/vsa.h.
//
// Argument checks run first and return before any CUDA call, so a rejected
// call launches nothing.  Device-detected errors land in one status word per
// device (a __device__ variable of this library); vsa_get_status reads and
// clears it.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "kernels.h"
#include "vsa.h"

struct vsa_plan {
  vsa::Geo g;
};

namespace {

__device__ unsigned int g_status_word;

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int rc = VSA_OK;
  int num_sms = 0;
  unsigned int* status = nullptr;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// Per-device set-up on first use with that device current: check the
// architecture (sm_100), count SMs and find the status word's address.
int device_state(DeviceState** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return VSA_ERR_NO_DEVICE;
  }
  if (dev >= kMaxDevices) return VSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return VSA_ERR_CUDA;
    }
    if (major != 10 || minor != 0) {
      s.rc = VSA_ERR_UNSUPPORTED;
    } else {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess) {
        cudaGetLastError();
        return VSA_ERR_CUDA;
      }
      s.status = static_cast<unsigned int*>(addr);
      s.num_sms = sms;
      s.rc = VSA_OK;
    }
    s.ready = true;
  }
  if (s.rc != VSA_OK) return s.rc;
  *out = &s;
  return VSA_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int log2i(int x) {
  int l = 0;
  while ((1 << l) < x) ++l;
  return l;
}

int check_dims(int B, int H, int D) {
  if (B < 1 || H < 1) return VSA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 65535) return VSA_ERR_UNSUPPORTED;
  if (D != 128) return VSA_ERR_UNSUPPORTED;
  return VSA_OK;
}

int from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return VSA_OK;
  return VSA_ERR_CUDA;
}

// Library-owned scratch of vsa_tile_coarse_static: the fused front end's
// 2 int32 arrival counters per (b, h), for at most kStaticMaxHeads heads
// (32 KB per device).  Its address is looked up once per device, with that
// device current.
constexpr int kStaticMaxHeads = 4096;
static __device__ __align__(256) int g_front_scratch[2 * kStaticMaxHeads];

struct StaticScratch {
  bool ready = false;
  int* ptr = nullptr;
};
std::mutex g_scratch_mu;
StaticScratch g_scratch[kMaxDevices];

int static_scratch(int** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return VSA_ERR_NO_DEVICE;
  }
  if (dev >= kMaxDevices) return VSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  StaticScratch& s = g_scratch[dev];
  if (!s.ready) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_front_scratch) != cudaSuccess || addr == nullptr) {
      cudaGetLastError();
      return VSA_ERR_CUDA;
    }
    s.ptr = static_cast<int*>(addr);
    s.ready = true;
  }
  *out = s.ptr;
  return VSA_OK;
}

}  // namespace

extern "C" {

int vsa_plan_create_prefix(int n_prefix, int T, int Hg, int Wg, int bt, int bh, int bw, vsa_plan_t* out) {
  if (!out) return VSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (n_prefix < 0 || T < 1 || Hg < 1 || Wg < 1 || bt < 1 || bh < 1 || bw < 1) return VSA_ERR_INVALID_ARG;
  if (!pow2(bt) || !pow2(bh) || !pow2(bw) || bw > 32) return VSA_ERR_UNSUPPORTED;
  const int bs = bt * bh * bw;
  if (bs != 64 && bs != 256) return VSA_ERR_UNSUPPORTED;
  vsa::Geo g;
  g.n_prefix = n_prefix;
  g.T = T;
  g.Hg = Hg;
  g.Wg = Wg;
  g.bt = bt;
  g.bh = bh;
  g.bw = bw;
  g.lbt = log2i(bt);
  g.lbh = log2i(bh);
  g.lbw = log2i(bw);
  g.bs = bs;
  g.lbs = log2i(bs);
  g.nT = (T + bt - 1) / bt;
  g.nH = (Hg + bh - 1) / bh;
  g.nW = (Wg + bw - 1) / bw;
  g.n_pre = (n_prefix + bs - 1) / bs;
  const long long nvid = static_cast<long long>(g.nT) * g.nH * g.nW;
  if (nvid + g.n_pre > (1 << 24)) return VSA_ERR_UNSUPPORTED;
  g.NB = static_cast<int>(nvid + g.n_pre);
  g.S = static_cast<long long>(n_prefix) + static_cast<long long>(T) * Hg * Wg;
  g.Sp = static_cast<long long>(g.NB) * bs;
  g.vfull = (T % bt == 0 && Hg % bh == 0 && Wg % bw == 0) ? 1 : 0;
  vsa_plan* p = new (std::nothrow) vsa_plan;
  if (!p) return VSA_ERR_INVALID_ARG;
  p->g = g;
  *out = p;
  return VSA_OK;
}

int vsa_plan_create(int T, int Hg, int Wg, int bt, int bh, int bw, vsa_plan_t* out) {
  return vsa_plan_create_prefix(0, T, Hg, Wg, bt, bh, bw, out);
}

void vsa_plan_destroy(vsa_plan_t plan) { delete plan; }

int vsa_plan_sizes(vsa_plan_t plan, int* num_blocks, int64_t* seq_len, int64_t* padded_len, int* block_tokens) {
  if (!plan) return VSA_ERR_INVALID_ARG;
  if (num_blocks) *num_blocks = plan->g.NB;
  if (seq_len) *seq_len = plan->g.S;
  if (padded_len) *padded_len = plan->g.Sp;
  if (block_tokens) *block_tokens = plan->g.bs;
  return VSA_OK;
}

int vsa_plan_describe(vsa_plan_t plan, int topk, char* buf, size_t n) {
  if (!plan || !buf || n == 0) return VSA_ERR_INVALID_ARG;
  const vsa::Geo& g = plan->g;
  if (topk < 1 || topk > g.NB) return VSA_ERR_TOPK;
  const double keep = 100.0 * topk / g.NB;
  int w;
  if (g.n_prefix > 0)
    w = std::snprintf(buf, n,
                      "seq_len=%lld, prefix_len=%d, dit_seq_shape=(%d, %d, %d), block_size=(%d, %d, %d), "
                      "num_blocks=%d, topk=%d, keep_ratio=%.1f%%",
                      g.S, g.n_prefix, g.T, g.Hg, g.Wg, g.bt, g.bh, g.bw, g.NB, topk, keep);
  else
    w = std::snprintf(buf, n,
                      "seq_len=%lld, dit_seq_shape=(%d, %d, %d), block_size=(%d, %d, %d), num_blocks=%d, "
                      "topk=%d, keep_ratio=%.1f%%",
                      g.S, g.T, g.Hg, g.Wg, g.bt, g.bh, g.bw, g.NB, topk, keep);
  return (w < 0 || static_cast<size_t>(w) >= n) ? VSA_ERR_INVALID_ARG : VSA_OK;
}

int vsa_tile_ex(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t* x, uint16_t* x_tiled, float* pooled, int B,
                int H, int D, vsa_stream_t stream) {
  if (!plan || !aligned16(x) || !aligned16(x_tiled)) return VSA_ERR_INVALID_ARG;
  if (pooled && !aligned16(pooled)) return VSA_ERR_INVALID_ARG;
  if (dtype != VSA_BF16 && dtype != VSA_F16) return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  return from_cuda(vsa::launch_tile(plan->g, B, H, x, x_tiled, pooled, dtype == VSA_F16,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

int vsa_tile(vsa_plan_t plan, const uint16_t* x, uint16_t* x_tiled, float* pooled, int B, int H, int D,
             vsa_stream_t stream) {
  return vsa_tile_ex(plan, VSA_BF16, x, x_tiled, pooled, B, H, D, stream);
}

int vsa_untile(vsa_plan_t plan, const uint16_t* x_tiled, uint16_t* x, int B, int H, int D, vsa_stream_t stream) {
  if (!plan || !aligned16(x) || !aligned16(x_tiled)) return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  return from_cuda(vsa::launch_untile(plan->g, B, H, x_tiled, x, reinterpret_cast<cudaStream_t>(stream)));
}

int vsa_coarse_topk(vsa_plan_t plan, const float* qbar, const float* kbar, int B, int H, int D, int topk,
                    int32_t* q2k_idx, int32_t* q2k_num, vsa_stream_t stream) {
  if (!plan || !aligned16(qbar) || !aligned16(kbar) || !aligned16(q2k_idx) || !aligned16(q2k_num))
    return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  const int NB = plan->g.NB;
  if (topk < 1 || topk > NB) return VSA_ERR_TOPK;
  if (NB > 2048) return VSA_ERR_UNSUPPORTED;  // scores of 8 rows must fit in shared memory
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  const vsa::SelectRule plain{topk, 0, nullptr};
  return from_cuda(vsa::launch_score_topk(B * H, NB, topk, plain, qbar, kbar, q2k_idx, q2k_num,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

namespace {
// The tile-64 selection's arguments: 0 < topk <= video blocks, a row stride
// that holds the longest row, an aligned (or absent) row-keep mask.
int check_prefix_rule(const vsa::Geo& g, int topk, int max_k, const uint8_t* row_keep) {
  if (topk < 1 || topk > g.NB - g.n_pre) return VSA_ERR_TOPK;
  if (max_k < (g.n_pre > 0 ? g.NB : topk)) return VSA_ERR_INVALID_ARG;
  if (row_keep && (reinterpret_cast<uintptr_t>(row_keep) & 15u)) return VSA_ERR_INVALID_ARG;
  if (g.NB > 2048) return VSA_ERR_UNSUPPORTED;  // scores of 8 rows must fit in shared memory
  return VSA_OK;
}
}  // namespace

int vsa_coarse_topk_prefix(vsa_plan_t plan, const float* qbar, const float* kbar, const uint8_t* row_keep, int B,
                           int H, int D, int topk, int max_k, int32_t* q2k_idx, int32_t* q2k_num,
                           vsa_stream_t stream) {
  if (!plan || !aligned16(qbar) || !aligned16(kbar) || !aligned16(q2k_idx) || !aligned16(q2k_num))
    return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  if (int rc = check_prefix_rule(plan->g, topk, max_k, row_keep)) return rc;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  const vsa::SelectRule rule{max_k, plan->g.n_pre, row_keep};
  return from_cuda(vsa::launch_score_topk(B * H, plan->g.NB, topk, rule, qbar, kbar, q2k_idx, q2k_num,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int vsa_coarse_compress(vsa_plan_t plan, const float* qbar, const float* kbar, const float* vbar, int B, int H,
                        int D, int topk, int32_t* q2k_idx, int32_t* q2k_num, float* o_compress, vsa_stream_t stream) {
  if (!plan || !aligned16(qbar) || !aligned16(kbar) || !aligned16(vbar) || !aligned16(o_compress))
    return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  const int NB = plan->g.NB;
  if (topk < 0 || topk > NB) return VSA_ERR_TOPK;
  if (topk > 0 && (!aligned16(q2k_idx) || !aligned16(q2k_num))) return VSA_ERR_INVALID_ARG;
  if (topk == 0 && (q2k_idx || q2k_num)) return VSA_ERR_INVALID_ARG;
  if (NB > 2048) return VSA_ERR_UNSUPPORTED;  // scores of 8 rows must fit in shared memory
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  return from_cuda(vsa::launch_coarse_compress(B * H, NB, topk, qbar, kbar, vbar, q2k_idx, q2k_num, o_compress,
                                               scale, reinterpret_cast<cudaStream_t>(stream)));
}

int vsa_tile_coarse(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    int B, int H, int D, int topk, uint16_t* q_tiled, uint16_t* k_tiled, uint16_t* v_tiled,
                    float* qbar, float* kbar, float* vbar, int32_t* q2k_idx, int32_t* q2k_num, float* o_compress,
                    int32_t* workspace, vsa_stream_t stream) {
  if (dtype != VSA_BF16 && dtype != VSA_F16) return VSA_ERR_INVALID_ARG;
  if (!plan || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_tiled) || !aligned16(k_tiled) ||
      !aligned16(v_tiled) || !aligned16(qbar) || !aligned16(kbar) || !aligned16(workspace))
    return VSA_ERR_INVALID_ARG;
  if ((vbar == nullptr) != (o_compress == nullptr)) return VSA_ERR_INVALID_ARG;
  if (vbar && (!aligned16(vbar) || !aligned16(o_compress))) return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  const int NB = plan->g.NB;
  if (topk < 0 || topk > NB) return VSA_ERR_TOPK;
  if (topk > 0 && (!aligned16(q2k_idx) || !aligned16(q2k_num))) return VSA_ERR_INVALID_ARG;
  if (topk == 0 && (q2k_idx || q2k_num)) return VSA_ERR_INVALID_ARG;
  if (NB > 2048) return VSA_ERR_UNSUPPORTED;  // scores of 8 rows must fit in shared memory
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  vsa::FrontArgs a;
  a.g = plan->g;
  a.H = H;
  a.BH = B * H;
  a.topk = topk;
  a.rule = vsa::SelectRule{topk, 0, nullptr};
  a.q = reinterpret_cast<const uint4*>(q);
  a.k = reinterpret_cast<const uint4*>(k);
  a.v = reinterpret_cast<const uint4*>(v);
  a.qt = reinterpret_cast<uint4*>(q_tiled);
  a.kt = reinterpret_cast<uint4*>(k_tiled);
  a.vt = reinterpret_cast<uint4*>(v_tiled);
  a.qbar = qbar;
  a.kbar = kbar;
  a.vbar = vbar;
  a.idx = q2k_idx;
  a.num = q2k_num;
  a.o_compress = o_compress;
  a.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  a.arrive = workspace;
  a.done = workspace + static_cast<long long>(B) * H;
  a.status = ds->status;
  a.f16 = dtype == VSA_F16;
  return from_cuda(vsa::launch_front(a, reinterpret_cast<cudaStream_t>(stream)));
}

int vsa_tile_coarse_prefix(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, const uint8_t* row_keep, int B, int H, int D, int topk, int max_k,
                           uint16_t* q_tiled, uint16_t* k_tiled, uint16_t* v_tiled, float* qbar, float* kbar,
                           int32_t* q2k_idx, int32_t* q2k_num, int32_t* workspace, vsa_stream_t stream) {
  if (dtype != VSA_BF16 && dtype != VSA_F16) return VSA_ERR_INVALID_ARG;
  if (!plan || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_tiled) || !aligned16(k_tiled) ||
      !aligned16(v_tiled) || !aligned16(qbar) || !aligned16(kbar) || !aligned16(workspace) ||
      !aligned16(q2k_idx) || !aligned16(q2k_num))
    return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  if (int rc = check_prefix_rule(plan->g, topk, max_k, row_keep)) return rc;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  vsa::FrontArgs a;
  a.g = plan->g;
  a.H = H;
  a.BH = B * H;
  a.topk = topk;
  a.rule = vsa::SelectRule{max_k, plan->g.n_pre, row_keep};
  a.q = reinterpret_cast<const uint4*>(q);
  a.k = reinterpret_cast<const uint4*>(k);
  a.v = reinterpret_cast<const uint4*>(v);
  a.qt = reinterpret_cast<uint4*>(q_tiled);
  a.kt = reinterpret_cast<uint4*>(k_tiled);
  a.vt = reinterpret_cast<uint4*>(v_tiled);
  a.qbar = qbar;
  a.kbar = kbar;
  a.vbar = nullptr;
  a.idx = q2k_idx;
  a.num = q2k_num;
  a.o_compress = nullptr;
  a.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  a.arrive = workspace;
  a.done = workspace + static_cast<long long>(B) * H;
  a.status = ds->status;
  a.f16 = dtype == VSA_F16;
  return from_cuda(vsa::launch_front(a, reinterpret_cast<cudaStream_t>(stream)));
}

int vsa_tile_coarse_static(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, int B, int H, int D, int topk, uint16_t* q_tiled, uint16_t* k_tiled,
                           uint16_t* v_tiled, float* qbar, float* kbar, float* vbar, int32_t* q2k_idx,
                           int32_t* q2k_num, float* o_compress, vsa_stream_t stream) {
  // the checks of vsa_tile_coarse, so that a rejected call touches no device memory
  if (dtype != VSA_BF16 && dtype != VSA_F16) return VSA_ERR_INVALID_ARG;
  if (!plan || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_tiled) || !aligned16(k_tiled) ||
      !aligned16(v_tiled) || !aligned16(qbar) || !aligned16(kbar))
    return VSA_ERR_INVALID_ARG;
  if ((vbar == nullptr) != (o_compress == nullptr)) return VSA_ERR_INVALID_ARG;
  if (vbar && (!aligned16(vbar) || !aligned16(o_compress))) return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  if (static_cast<long long>(B) * H > kStaticMaxHeads) return VSA_ERR_UNSUPPORTED;
  const int NB = plan->g.NB;
  if (topk < 0 || topk > NB) return VSA_ERR_TOPK;
  if (topk > 0 && (!aligned16(q2k_idx) || !aligned16(q2k_num))) return VSA_ERR_INVALID_ARG;
  if (topk == 0 && (q2k_idx || q2k_num)) return VSA_ERR_INVALID_ARG;
  if (NB > 2048) return VSA_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  int* scratch = nullptr;
  if (int rc = static_scratch(&scratch)) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the counters must start at zero (a call that timed out may leave them set)
  if (cudaMemsetAsync(scratch, 0, sizeof(int) * 2 * static_cast<size_t>(B) * H, s) != cudaSuccess) {
    cudaGetLastError();
    return VSA_ERR_CUDA;
  }
  return vsa_tile_coarse(plan, dtype, q, k, v, B, H, D, topk, q_tiled, k_tiled, v_tiled, qbar, kbar, vbar, q2k_idx,
                         q2k_num, o_compress, scratch, stream);
}

int vsa_untile_gate(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t* o_tiled, const float* o_compress,
                    const uint16_t* gate, uint16_t* o, int B, int H, int D, vsa_stream_t stream) {
  if (dtype != VSA_BF16 && dtype != VSA_F16) return VSA_ERR_INVALID_ARG;
  if (!plan || !aligned16(o_tiled) || !aligned16(o_compress) || !aligned16(gate) || !aligned16(o))
    return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  return from_cuda(vsa::launch_untile_gate(plan->g, B, H, o_tiled, o_compress, gate, o, dtype == VSA_F16,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

int vsa_map_to_index(const uint8_t* map, int B, int H, int NQ, int NK, int32_t* q2k_idx, int32_t* q2k_num,
                     vsa_stream_t stream) {
  if (!map || !aligned16(q2k_idx) || !aligned16(q2k_num)) return VSA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || NQ < 1 || NK < 1) return VSA_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * H * NQ;
  if (rows > (1ll << 34)) return VSA_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  return from_cuda(vsa::launch_map_to_index(map, rows, NK, q2k_idx, q2k_num, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {
int sparse_attn_fwd_impl(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const int32_t* q2k_idx, const int32_t* q2k_num, int max_k, int B, int H,
                         int D, uint16_t* o, float* lse, int32_t* queue, vsa_stream_t stream) {
  if (dtype != VSA_BF16 && dtype != VSA_F16) return VSA_ERR_INVALID_ARG;
  if (!plan || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return VSA_ERR_INVALID_ARG;
  if (!aligned16(q2k_idx) || !aligned16(q2k_num) || max_k < 1) return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  const vsa::Geo& g = plan->g;
  if (g.bs == 64 && (g.NB & 1)) return VSA_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  vsa::AttnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.idx = q2k_idx;
  a.num = q2k_num;
  a.max_k = max_k;
  a.BH = B * H;
  a.o = o;
  a.lse = lse;
  a.status = ds->status;
  a.num_sms = ds->num_sms;
  a.f16 = dtype == VSA_F16;
  a.queue = queue;
  return from_cuda(vsa::launch_attn_fwd(g, a, reinterpret_cast<cudaStream_t>(stream)));
}
}  // namespace

int vsa_sparse_attn_fwd_ex(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, const int32_t* q2k_idx, const int32_t* q2k_num, int max_k, int B, int H,
                           int D, uint16_t* o, float* lse, vsa_stream_t stream) {
  return sparse_attn_fwd_impl(plan, dtype, q, k, v, q2k_idx, q2k_num, max_k, B, H, D, o, lse, nullptr, stream);
}

int vsa_sparse_attn_fwd_ws(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, const int32_t* q2k_idx, const int32_t* q2k_num, int max_k, int B, int H,
                           int D, uint16_t* o, float* lse, int32_t* workspace, vsa_stream_t stream) {
  if (!aligned16(workspace)) return VSA_ERR_INVALID_ARG;
  return sparse_attn_fwd_impl(plan, dtype, q, k, v, q2k_idx, q2k_num, max_k, B, H, D, o, lse, workspace, stream);
}

int vsa_sparse_attn_fwd(vsa_plan_t plan, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const int32_t* q2k_idx, const int32_t* q2k_num, int max_k, int B, int H, int D, uint16_t* o,
                        float* lse, vsa_stream_t stream) {
  return vsa_sparse_attn_fwd_ex(plan, VSA_BF16, q, k, v, q2k_idx, q2k_num, max_k, B, H, D, o, lse, stream);
}

int vsa_quantize_nvfp4(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t* x_tiled, int B, int H, int D,
                       uint8_t* codes, uint8_t* scales, vsa_stream_t stream) {
  if (dtype != VSA_BF16 && dtype != VSA_F16) return VSA_ERR_INVALID_ARG;
  if (!plan || !aligned16(x_tiled) || !aligned16(codes) || !aligned16(scales)) return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  const vsa::Geo& g = plan->g;
  if (g.Sp % 128 != 0) return VSA_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  const long long rows = static_cast<long long>(B) * H * g.Sp;
  return from_cuda(vsa::launch_quant_nvfp4(rows, x_tiled, codes, scales, dtype == VSA_F16,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

namespace {
int sparse_attn_fwd_nvfp4_impl(vsa_plan_t plan, vsa_dtype_t dtype, const uint8_t* q_codes, const uint8_t* q_scales,
                               const uint8_t* k_codes, const uint8_t* k_scales, const uint16_t* v,
                               const int32_t* q2k_idx, const int32_t* q2k_num, int max_k, int B, int H, int D,
                               uint16_t* o, float* lse, int32_t* queue, vsa_stream_t stream) {
  if (dtype != VSA_BF16 && dtype != VSA_F16) return VSA_ERR_INVALID_ARG;
  if (!plan || !aligned16(q_codes) || !aligned16(q_scales) || !aligned16(k_codes) || !aligned16(k_scales) ||
      !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return VSA_ERR_INVALID_ARG;
  if (!aligned16(q2k_idx) || !aligned16(q2k_num) || max_k < 1) return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  const vsa::Geo& g = plan->g;
  if (g.Sp % 128 != 0) return VSA_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  vsa::AttnFp4Args a;
  a.q = q_codes;
  a.q_sf = q_scales;
  a.k = k_codes;
  a.k_sf = k_scales;
  a.v = v;
  a.idx = q2k_idx;
  a.num = q2k_num;
  a.max_k = max_k;
  a.BH = B * H;
  a.o = o;
  a.lse = lse;
  a.status = ds->status;
  a.num_sms = ds->num_sms;
  a.f16 = dtype == VSA_F16;
  a.queue = queue;
  return from_cuda(vsa::launch_attn_fwd_nvfp4(g, a, reinterpret_cast<cudaStream_t>(stream)));
}
}  // namespace

int vsa_sparse_attn_fwd_nvfp4(vsa_plan_t plan, vsa_dtype_t dtype, const uint8_t* q_codes, const uint8_t* q_scales,
                              const uint8_t* k_codes, const uint8_t* k_scales, const uint16_t* v,
                              const int32_t* q2k_idx, const int32_t* q2k_num, int max_k, int B, int H, int D,
                              uint16_t* o, float* lse, vsa_stream_t stream) {
  return sparse_attn_fwd_nvfp4_impl(plan, dtype, q_codes, q_scales, k_codes, k_scales, v, q2k_idx, q2k_num, max_k,
                                    B, H, D, o, lse, nullptr, stream);
}

int vsa_sparse_attn_fwd_nvfp4_ws(vsa_plan_t plan, vsa_dtype_t dtype, const uint8_t* q_codes, const uint8_t* q_scales,
                                 const uint8_t* k_codes, const uint8_t* k_scales, const uint16_t* v,
                                 const int32_t* q2k_idx, const int32_t* q2k_num, int max_k, int B, int H, int D,
                                 uint16_t* o, float* lse, int32_t* workspace, vsa_stream_t stream) {
  if (!aligned16(workspace)) return VSA_ERR_INVALID_ARG;
  return sparse_attn_fwd_nvfp4_impl(plan, dtype, q_codes, q_scales, k_codes, k_scales, v, q2k_idx, q2k_num, max_k,
                                    B, H, D, o, lse, workspace, stream);
}

int vsa_sparse_attn_bwd_workspace(vsa_plan_t plan, int B, int H, int max_k, size_t* bytes) {
  if (!plan || !bytes || B < 1 || H < 1 || max_k < 1) return VSA_ERR_INVALID_ARG;
  *bytes = vsa::attn_bwd_workspace_bytes(plan->g, B * H, max_k);
  return VSA_OK;
}

int vsa_sparse_attn_bwd(vsa_plan_t plan, vsa_dtype_t dtype, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const uint16_t* o, const float* lse, const uint16_t* dO, const int32_t* q2k_idx,
                        const int32_t* q2k_num, int max_k, int B, int H, int D, uint16_t* dq, uint16_t* dk,
                        uint16_t* dv, void* workspace, vsa_stream_t stream) {
  if (dtype != VSA_BF16 && dtype != VSA_F16) return VSA_ERR_INVALID_ARG;
  if (!plan || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return VSA_ERR_INVALID_ARG;
  if (!aligned16(q2k_idx) || !aligned16(q2k_num) || max_k < 1) return VSA_ERR_INVALID_ARG;
  if (int rc = check_dims(B, H, D)) return rc;
  const vsa::Geo& g = plan->g;
  if (g.NB > vsa::kBwdMaxBlocks) return VSA_ERR_UNSUPPORTED;  // transposed selection in shared memory
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  vsa::AttnBwdArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.dO = dO;
  a.lse = lse;
  a.idx = q2k_idx;
  a.num = q2k_num;
  a.max_k = max_k;
  a.BH = B * H;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.workspace = workspace;
  a.status = ds->status;
  a.f16 = dtype == VSA_F16;
  return from_cuda(vsa::launch_attn_bwd(g, a, reinterpret_cast<cudaStream_t>(stream)));
}

int vsa_get_status(vsa_stream_t stream, int* device_status) {
  if (!device_status) return VSA_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if (int rc = device_state(&ds)) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return VSA_ERR_CUDA;
  if (cudaMemcpyAsync(&v, ds->status, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return VSA_ERR_CUDA;
  if (cudaMemsetAsync(ds->status, 0, sizeof(unsigned int), s) != cudaSuccess) return VSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return VSA_ERR_CUDA;
  *device_status = static_cast<int>(v);
  return VSA_OK;
}

const char* vsa_strerror(int status) {
  switch (status) {
    case VSA_OK: return "ok";
    case VSA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size)";
    case VSA_ERR_UNSUPPORTED: return "unsupported configuration (head size, block size, device)";
    case VSA_ERR_TOPK: return "topk must satisfy 0 < topk <= num_blocks";
    case VSA_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case VSA_ERR_BAD_INDEX: return "device: block id outside [0, num_blocks) or count outside [0, max_k]";
    case VSA_ERR_TIMEOUT: return "device: a pipeline wait ran out and the kernel stopped early";
    case VSA_ERR_NO_DEVICE: return "no usable CUDA device";
    default: return "unknown status";
  }
}

}  // extern "C"
