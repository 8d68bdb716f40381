// api.cu -- the C ABI of libhaste.so (declared in include/haste.h): plan builder,
// argument checks, workspace layout and the launch sequences of the calls.
//
// The library is built as one translation unit (this file includes the kernel
// sources) so that the device error word is a single static device variable.
#include "../../include/haste.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include "head.cu"
#include "tail.cu"
#include "tail_v2.cu"
#include "dx_band.cu"
#include "tail_given.cu"
#include "topk.cu"
#include "plan.cu"

using namespace haste;

struct haste_plan_s {
  int64_t n_groups;
  int32_t G, k, d;
  int device;
  int32_t* idx_d;
  int32_t* inv_off_d;
  int32_t* inv_ent_d;
  int32_t* scratch_d;  // counting-sort scratch of the device build (NULL: built on the host)
  int32_t* upd_d;      // staging of haste_plan_update: changed group ids and rows
  size_t upd_cap;      // ints of upd_d
};

namespace {

thread_local std::string g_err;

haste_status_t fail(haste_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

haste_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(HASTE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define HASTE_CUDA(call)                                       \
  do {                                                         \
    cudaError_t e_ = (call);                                   \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call);        \
  } while (0)

inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }
inline int elem_bytes(haste_dtype_t dt) { return dt == HASTE_F32 ? 4 : 2; }
inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

struct DeviceInfo {
  int sms = 0, smem_optin = 0, major = 0;
};

haste_status_t device_info(DeviceInfo& di) {
  int dev = 0;
  HASTE_CUDA(cudaGetDevice(&dev));
  HASTE_CUDA(cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev));
  HASTE_CUDA(cudaDeviceGetAttribute(&di.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
  HASTE_CUDA(cudaDeviceGetAttribute(&di.major, cudaDevAttrComputeCapabilityMajor, dev));
  if (di.major != 10) return fail(HASTE_ERR_CUDA, "libhaste needs an sm_100 GPU (found compute capability %d.x)", di.major);
  return HASTE_OK;
}

// Per-launch CUDA events on the launching stream while profiling is on
// (haste_profile_start / haste_profile_stop).
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
struct ProfState {
  bool on = false;
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> pool;
  size_t next = 0;
  std::mutex mu;
};
ProfState g_prof;

cudaEvent_t prof_event() {
  if (g_prof.next < g_prof.pool.size()) return g_prof.pool[g_prof.next++];
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  g_prof.pool.push_back(e);
  ++g_prof.next;
  return e;
}

// Brackets one kernel launch with events when profiling is on.
class ProfScope {
 public:
  ProfScope(const char* name, cudaStream_t s) : name_(name), s_(s) {
    if (!g_prof.on) return;
    std::lock_guard<std::mutex> g(g_prof.mu);
    a_ = prof_event();
    if (a_) cudaEventRecord(a_, s_);
  }
  ~ProfScope() {
    if (!g_prof.on || !a_) return;
    std::lock_guard<std::mutex> g(g_prof.mu);
    cudaEvent_t b = prof_event();
    if (!b) return;
    cudaEventRecord(b, s_);
    g_prof.recs.push_back({name_, a_, b});
  }

 private:
  const char* name_;
  cudaStream_t s_;
  cudaEvent_t a_ = nullptr;
};

// Tiling of the dX pass.  ns > 0: the pipelined band-product kernel (k_dx_band)
// with an ns-stage ring, one CTA per (group chunk, feature band of up to 256,
// batch half of up to 256 rows); ns = 0: the staged kernel, feature bands sized
// so the fp32 band accumulator fits in shared memory.  Group chunks: as many as
// keep every CTA resident.
struct DxTiling {
  int band, n_bands, n_chunks, ns, n_halves;
};

// The warp-specialised TMA kernels cover bf16 with G in {16, 32, 64} and k in
// {64, 128}: the fused step kernel up to two 128-row batch tiles, the dX pass up
// to four; other shapes run the staged kernels of tail.cu.
bool use_v2(const haste_plan_s& p, int Bp, int elem) { return elem == 2 && tail2::supported(p.G, p.k, Bp); }
bool use_dx_band(const haste_plan_s& p, int Bp, int elem) { return elem == 2 && tail2::dx_supported(p.G, p.k, Bp); }

DxTiling dx_tiling(const haste_plan_s& p, int Bp, int elem, int sms, int smem_optin) {
  DxTiling t{};
  const int kHeadroom = 4096;  // static shared memory and launch reserve
  int per_chunk;
  if (use_dx_band(p, Bp, elem) &&
      tail2::dx_config(p.G, p.k, p.d, Bp, (size_t)smem_optin, kHeadroom, &t.band, &t.n_bands, &t.ns)) {
    t.n_halves = (Bp + 255) / 256;
    per_chunk = t.n_bands * t.n_halves;  // a CTA covers up to 256 batch rows of its band
  } else {
    const long avail = (long)smem_optin - (long)tail::smem_dx(elem, p.k, p.G, 0) - kHeadroom;
    int band = (int)std::min<long>(256, avail / 512);
    band = std::max(8, band & ~7);
    if (band > p.d) band = round_up(p.d, 8);
    // as few bands as fit, then split d evenly between them
    t.n_bands = (p.d + band - 1) / band;
    t.band = round_up((p.d + t.n_bands - 1) / t.n_bands, 8);
    t.ns = 0;
    per_chunk = (Bp / 128) * t.n_bands;
  }
  int c = std::max(1, sms / per_chunk);
  // chunks of whole ring items (super-groups of 64 labels) for the band kernel
  const int64_t units = t.ns > 0 ? tail2::dx_items(p.n_groups, p.G) : p.n_groups;
  if ((int64_t)c > units) c = (int)units;
  t.n_chunks = c;
  return t;
}

// Workspace layout of the tail calls.
struct TailWs {
  size_t xt, dx_part, dy_buf, loss_part, total;
};

constexpr int kMaxLossParts = 4096;

TailWs tail_ws(const haste_plan_s& p, int B, int elem, const DxTiling& t) {
  TailWs w{};
  const int Bp = round_up(B, 128);
  size_t off = 0;
  w.xt = off;
  off = align256(off + (size_t)p.d * Bp * elem);
  w.dx_part = off;
  off = align256(off + (size_t)t.n_chunks * p.d * Bp * 4);
  // [B, L] (staged kernels) or the fused step's buffer [n_items * 64][Bp]: items
  // of 64 / G groups, whose 64 labels cover the G-wide groups (the last item may
  // be partial)
  w.dy_buf = off;
  size_t dy_elems = (size_t)Bp * p.n_groups * p.G;
  if (p.G <= 64 && 64 % p.G == 0) dy_elems = std::max(dy_elems, (size_t)tail2::dx_items(p.n_groups, p.G) * Bp * 64);
  off = align256(off + dy_elems * elem);
  w.loss_part = off;
  off = align256(off + (size_t)kMaxLossParts * 4);
  w.total = off;
  return w;
}

// A plan's arrays live on the device that was current when it was built; a call
// on another device would read them through peer access or fault.
haste_status_t check_plan_device(const haste_plan_s* p) {
  if (!p) return fail(HASTE_ERR_INVALID_ARG, "plan is NULL");
  int dev = -1;
  HASTE_CUDA(cudaGetDevice(&dev));
  if (dev != p->device)
    return fail(HASTE_ERR_INVALID_ARG, "the plan was built on device %d, but device %d is current", p->device, dev);
  return HASTE_OK;
}

haste_status_t check_tail(const haste_plan_s* p, int B, haste_dtype_t dt, const DeviceInfo& di) {
  if (!p) return fail(HASTE_ERR_INVALID_ARG, "plan is NULL");
  if (haste_status_t st = check_plan_device(p)) return st;
  if (dt != HASTE_F32 && dt != HASTE_BF16) return fail(HASTE_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  if (B <= 0) return fail(HASTE_ERR_INVALID_ARG, "B must be positive (got %d)", B);
  const int E = elem_bytes(dt);
  if ((p->k * E) % 128 || p->k > 256)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "k=%d: the GPU path needs k*elem %% 128 == 0 and k <= 256", p->k);
  if (p->G % 16 || p->G < 16 || p->G > 128)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "G=%d: the GPU path needs G %% 16 == 0 and 16 <= G <= 128", p->G);
  const int64_t L = p->n_groups * p->G;
  if ((L * E) % 16) return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "L*elem must be a multiple of 16 bytes");
  if (B > 512) return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "B=%d: the GPU path supports B <= 512", B);
  const int Bp = round_up(B, 128);
  const size_t need = std::max(std::max(tail::smem_forward(E, p->k, p->G), tail::smem_dw(E, p->k, p->G, Bp)),
                               tail::smem_dx(E, p->k, p->G, 8));
  if (need > (size_t)di.smem_optin)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "tiles need %zu bytes of shared memory (> %d)", need, di.smem_optin);
  return HASTE_OK;
}

haste_status_t check_ws(void* ws, size_t have, size_t need) {
  if (have < need) return fail(HASTE_ERR_WORKSPACE, "workspace of %zu bytes is below the %zu needed", have, need);
  if (need && !ws) return fail(HASTE_ERR_INVALID_ARG, "workspace pointer is NULL");
  return HASTE_OK;
}

TailArgs make_args(const haste_plan_s& p, int B) {
  TailArgs a{};
  a.sh.B = B;
  a.sh.Bp = round_up(B, 128);
  a.sh.d = p.d;
  a.sh.G = p.G;
  a.sh.k = p.k;
  a.sh.n_groups = p.n_groups;
  a.sh.L = p.n_groups * p.G;
  a.idx = p.idx_d;
  return a;
}

// dX pass through a pipelined bf16 kernel, from the caller's row-major [B, L]
// gradient or from the fused step's buffer of label rows [n_items * 64][Bp].
cudaError_t dx_v2(const haste_plan_s& p, int B, const void* W, const void* dY, bool group_major, float* part,
                  const DxTiling& t, cudaStream_t s) {
  v2::DxArgs a{};
  a.sh = make_args(p, B).sh;
  a.idx = p.idx_d;
  a.dY = static_cast<const __nv_bfloat16*>(dY);
  a.W = static_cast<const __nv_bfloat16*>(W);
  a.dX_part = part;
  a.band = t.band;
  a.n_bands = t.n_bands;
  a.n_halves = t.n_halves;
  a.n_chunks = t.n_chunks;
  a.ns = t.ns;
  a.group_major = group_major ? 1 : 0;
  return tail2::launch_dx(p.G, p.k, a, dY, W, s);
}

template <typename T>
cudaError_t xt(const TailArgs& a, const void* X, void* Xt, cudaStream_t st) {
  return tail::launch_xt<T>(X, Xt, a.sh.B, a.sh.Bp, a.sh.d, st);
}

// Scratch of haste_backward_dx_noalloc: static device memory (no allocation at
// call time).  Holds the per-chunk dX partials; every GPU that loads the library
// keeps these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device (host code only
// sees a host-side stand-in under that name).
constexpr int kMaxDevices = 64;
void* g_noalloc_addr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

haste_status_t noalloc_scratch(void** out) {
  int dev = 0;
  HASTE_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(HASTE_ERR_INVALID_ARG, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    HASTE_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return HASTE_OK;
}

// Validation of index rows (host [n_rows, k]): the first offending element in
// row-major order decides: out of [0, d) -> HASTE_ERR_INDEX_OUT_OF_RANGE, not
// above its predecessor -> HASTE_ERR_INDEX_UNSORTED_OR_DUP.  `what` names the
// rows in the message.  Split over threads by contiguous row ranges.
haste_status_t validate_rows(const int32_t* idx, int64_t n_rows, int32_t k, int32_t d, const char* what) {
  const unsigned hw = std::thread::hardware_concurrency();
  const int nt = (int)std::min<int64_t>(std::max(1u, std::min(hw, 32u)), std::max<int64_t>(1, n_rows * k / (1 << 16)));
  std::vector<int64_t> bad(nt, -1);
  std::vector<int> code(nt, 0);
  auto scan = [&](int t) {
    for (int64_t r = n_rows * t / nt; r < n_rows * (t + 1) / nt; ++r) {
      int32_t prev = -1;
      for (int32_t s = 0; s < k; ++s) {
        const int32_t f = idx[r * k + s];
        if ((uint32_t)f >= (uint32_t)d || f <= prev) {
          bad[t] = r * k + s;
          code[t] = (uint32_t)f >= (uint32_t)d ? HASTE_ERR_INDEX_OUT_OF_RANGE : HASTE_ERR_INDEX_UNSORTED_OR_DUP;
          return;
        }
        prev = f;
      }
    }
  };
  std::vector<std::thread> th;
  for (int t = 1; t < nt; ++t) th.emplace_back(scan, t);
  scan(0);
  for (auto& x : th) x.join();
  for (int t = 0; t < nt; ++t)
    if (bad[t] >= 0)
      return fail((haste_status_t)code[t], "%s element %lld (row %lld, slot %lld) is %s", what, (long long)bad[t],
                  (long long)(bad[t] / k), (long long)(bad[t] % k),
                  code[t] == HASTE_ERR_INDEX_OUT_OF_RANGE ? "out of [0, d)" : "not above its predecessor");
  return HASTE_OK;
}

// The device build needs the d feature counters of a chunk in shared memory.
bool device_build_fits(int d, int smem_optin) { return (size_t)d * 4 + 1024 <= (size_t)smem_optin; }

}  // namespace

extern "C" {

int haste_abi_version(void) { return 1; }

const char* haste_last_error(void) { return g_err.c_str(); }

haste_status_t haste_device_status(haste_stream_t stream) {
  HASTE_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int v = 0;
  HASTE_CUDA(cudaMemcpyFromSymbol(&v, g_device_error, sizeof v));
  if (v != 0) {
    const int zero = 0;
    HASTE_CUDA(cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero));
    return fail(HASTE_ERR_TIMEOUT, "a kernel's bounded wait ran out (device error word %d)", v);
  }
  return HASTE_OK;
}

haste_status_t haste_profile_start(void) {
  std::lock_guard<std::mutex> g(g_prof.mu);
  g_prof.recs.clear();
  g_prof.next = 0;
  g_prof.on = true;
  return HASTE_OK;
}

int32_t haste_profile_stop(haste_kernel_time_t* out, int32_t max_entries) {
  std::lock_guard<std::mutex> g(g_prof.mu);
  g_prof.on = false;
  std::vector<haste_kernel_time_t> agg;
  for (const ProfRec& r : g_prof.recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return -1;
    auto it = std::find_if(agg.begin(), agg.end(), [&](const haste_kernel_time_t& k) { return !strcmp(k.name, r.name); });
    if (it == agg.end()) {
      agg.push_back({r.name, 1, (double)ms});
    } else {
      it->launches += 1;
      it->total_ms += ms;
    }
  }
  g_prof.recs.clear();
  g_prof.next = 0;
  const int32_t n = (int32_t)agg.size();
  for (int32_t i = 0; out && i < n && i < max_entries; ++i) out[i] = agg[i];
  return n;
}

haste_status_t haste_set_wait_limit_ns(uint64_t ns) {
  const uint64_t v = ns ? ns : kWaitLimitNs;
  if (v > kWaitLimitNs) return fail(HASTE_ERR_INVALID_ARG, "wait limit %llu ns above the default %llu ns",
                                    (unsigned long long)v, (unsigned long long)kWaitLimitNs);
  HASTE_CUDA(cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof v));
  return HASTE_OK;
}

haste_status_t haste_selftest_wait_timeout(haste_stream_t stream) {
  DeviceInfo di;
  haste_status_t st = device_info(di);
  if (st != HASTE_OK) return st;
  cudaError_t e = tail::launch_selftest_wait(20000000ull, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HASTE_OK : cuda_fail(e, "haste_selftest_wait_timeout launch");
}

// Validation plus a stable counting sort of the entries by feature, split over
// threads by contiguous group ranges: per-thread feature histograms, a prefix
// over (feature, thread) in that order, then each thread scatters its own range.
// Entries of one feature therefore land in ascending group order.
haste_status_t haste_plan_inverse_host(const int32_t* idx, int64_t n_groups, int32_t k, int32_t d,
                                       int32_t* inv_off, int32_t* inv_ent) {
  if (!idx || !inv_off || !inv_ent) return fail(HASTE_ERR_INVALID_ARG, "NULL pointer");
  if (n_groups <= 0 || k <= 0 || d <= 0) return fail(HASTE_ERR_INVALID_ARG, "n_groups, k and d must be positive");
  if (n_groups * (int64_t)k > 0x7fffffffLL)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "n_groups*k must fit in int32");
  const int64_t n = n_groups * (int64_t)k;
  unsigned hw = std::thread::hardware_concurrency();
  int nt = (int)std::min<int64_t>(std::max(1u, std::min(hw, 32u)), std::max<int64_t>(1, n / (1 << 16)));
  std::vector<int64_t> bounds(nt + 1);
  for (int t = 0; t <= nt; ++t) bounds[t] = n_groups * t / nt;
  std::vector<std::vector<int32_t>> hist(nt, std::vector<int32_t>(d, 0));
  std::vector<int64_t> bad(nt, -1);  // first offending flat position per thread
  std::vector<int> bad_code(nt, 0);

  auto count = [&](int t) {
    std::vector<int32_t>& h = hist[t];
    for (int64_t g = bounds[t]; g < bounds[t + 1]; ++g) {
      const int32_t* row = idx + g * k;
      int32_t prev = -1;
      for (int32_t s = 0; s < k; ++s) {
        const int32_t f = row[s];
        if ((uint32_t)f >= (uint32_t)d) {
          bad[t] = g * k + s;
          bad_code[t] = HASTE_ERR_INDEX_OUT_OF_RANGE;
          return;
        }
        if (f <= prev) {
          bad[t] = g * k + s;
          bad_code[t] = HASTE_ERR_INDEX_UNSORTED_OR_DUP;
          return;
        }
        prev = f;
        ++h[f];
      }
    }
  };
  {
    std::vector<std::thread> th;
    for (int t = 1; t < nt; ++t) th.emplace_back(count, t);
    count(0);
    for (auto& x : th) x.join();
  }
  for (int t = 0; t < nt; ++t)
    if (bad[t] >= 0)
      return fail((haste_status_t)bad_code[t], "idx element %lld (group %lld, slot %lld) is %s",
                  (long long)bad[t], (long long)(bad[t] / k), (long long)(bad[t] % k),
                  bad_code[t] == HASTE_ERR_INDEX_OUT_OF_RANGE ? "out of [0, d)" : "not above its predecessor");
  // prefix in (feature, thread) order: thread t's entries of feature f start at
  // inv_off[f] + sum of the earlier threads' counts of f
  int64_t run = 0;
  for (int32_t f = 0; f < d; ++f) {
    inv_off[f] = (int32_t)run;
    for (int t = 0; t < nt; ++t) {
      const int32_t c = hist[t][f];
      hist[t][f] = (int32_t)run;
      run += c;
    }
  }
  inv_off[d] = (int32_t)run;
  auto scatter = [&](int t) {
    std::vector<int32_t>& pos = hist[t];
    for (int64_t g = bounds[t]; g < bounds[t + 1]; ++g)
      for (int32_t s = 0; s < k; ++s) inv_ent[pos[idx[g * k + s]]++] = (int32_t)(g * k + s);
  };
  {
    std::vector<std::thread> th;
    for (int t = 1; t < nt; ++t) th.emplace_back(scatter, t);
    scatter(0);
    for (auto& x : th) x.join();
  }
  return HASTE_OK;
}

haste_status_t haste_plan(haste_plan_t* out, const int32_t* idx, int64_t n_groups, int32_t G, int32_t k, int32_t d,
                          haste_stream_t stream) {
  if (!out) return fail(HASTE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (G <= 0) return fail(HASTE_ERR_INVALID_ARG, "G must be positive");
  if (!idx) return fail(HASTE_ERR_INVALID_ARG, "NULL pointer");
  if (n_groups <= 0 || k <= 0 || d <= 0) return fail(HASTE_ERR_INVALID_ARG, "n_groups, k and d must be positive");
  if (n_groups * (int64_t)G > 0x7fffffffffffLL) return fail(HASTE_ERR_INVALID_ARG, "L too large");
  if (n_groups * (int64_t)k > 0x7fffffffLL) return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "n_groups*k must fit in int32");
  haste_status_t st = validate_rows(idx, n_groups, k, d, "idx");
  if (st != HASTE_OK) return st;
  DeviceInfo di;
  if ((st = device_info(di)) != HASTE_OK) return st;
  const int64_t n = n_groups * (int64_t)k;
  haste_plan_s* p = new haste_plan_s{};
  p->n_groups = n_groups;
  p->G = G;
  p->k = k;
  p->d = d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool on_device = device_build_fits(d, di.smem_optin);
  std::vector<int32_t> off, ent;
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = cudaMalloc(&p->idx_d, n * 4);
  if (e == cudaSuccess) e = cudaMalloc(&p->inv_off_d, ((size_t)d + 1) * 4);
  if (e == cudaSuccess) e = cudaMalloc(&p->inv_ent_d, n * 4);
  if (e == cudaSuccess && on_device) e = cudaMalloc(&p->scratch_d, plan::scratch_ints(n_groups, d) * 4);
  if (e == cudaSuccess) e = cudaMemcpyAsync(p->idx_d, idx, n * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && on_device) {
    e = plan::build_inverse(p->idx_d, n_groups, k, d, p->scratch_d, p->inv_off_d, p->inv_ent_d, s);
  } else if (e == cudaSuccess) {
    // wide d: the inverse map is built on the host and uploaded
    off.resize((size_t)d + 1);
    ent.resize((size_t)n);
    if ((st = haste_plan_inverse_host(idx, n_groups, k, d, off.data(), ent.data())) != HASTE_OK) {
      cudaStreamSynchronize(s);
      haste_plan_destroy(p);
      return st;
    }
    e = cudaMemcpyAsync(p->inv_off_d, off.data(), ((size_t)d + 1) * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(p->inv_ent_d, ent.data(), n * 4, cudaMemcpyHostToDevice, s);
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    haste_plan_destroy(p);
    return cuda_fail(e, "plan build");
  }
  *out = p;
  return HASTE_OK;
}

haste_status_t haste_plan_update(haste_plan_t p, const int32_t* groups, int64_t n_changed, const int32_t* rows,
                                 haste_stream_t stream) {
  haste_status_t st = check_plan_device(p);
  if (st != HASTE_OK) return st;
  if (n_changed < 0 || n_changed > p->n_groups) return fail(HASTE_ERR_INVALID_ARG, "n_changed out of [0, n_groups]");
  if (n_changed == 0) return HASTE_OK;
  if (!groups || !rows) return fail(HASTE_ERR_INVALID_ARG, "NULL pointer");
  if (!p->scratch_d)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "d=%d: the plan's inverse map is built on the host; rebuild the plan",
                p->d);
  for (int64_t i = 0; i < n_changed; ++i)
    if (groups[i] < 0 || groups[i] >= p->n_groups || (i > 0 && groups[i] <= groups[i - 1]))
      return fail(HASTE_ERR_INVALID_ARG, "groups[%lld] = %d: group ids must be ascending in [0, n_groups)",
                  (long long)i, groups[i]);
  if ((st = validate_rows(rows, n_changed, p->k, p->d, "rows")) != HASTE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t need = (size_t)n_changed * (p->k + 1);
  if (need > p->upd_cap) {
    HASTE_CUDA(cudaStreamSynchronize(s));  // an earlier update may still read the old staging
    cudaFree(p->upd_d);
    p->upd_d = nullptr;
    p->upd_cap = 0;
    HASTE_CUDA(cudaMalloc(&p->upd_d, need * 4));
    p->upd_cap = need;
  }
  int32_t* g_d = p->upd_d;
  int32_t* r_d = p->upd_d + n_changed;
  HASTE_CUDA(cudaMemcpyAsync(g_d, groups, (size_t)n_changed * 4, cudaMemcpyHostToDevice, s));
  HASTE_CUDA(cudaMemcpyAsync(r_d, rows, (size_t)n_changed * p->k * 4, cudaMemcpyHostToDevice, s));
  cudaError_t e;
  {
    ProfScope ps("plan_update", s);
    const int64_t tot = n_changed * p->k;
    plan::k_plan_set_rows<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(p->idx_d, p->k, g_d, r_d, n_changed);
    e = cudaGetLastError();
    if (e == cudaSuccess)
      e = plan::build_inverse(p->idx_d, p->n_groups, p->k, p->d, p->scratch_d, p->inv_off_d, p->inv_ent_d, s);
  }
  return e == cudaSuccess ? HASTE_OK : cuda_fail(e, "haste_plan_update launch");
}

haste_status_t haste_plan_destroy(haste_plan_t p) {
  if (!p) return HASTE_OK;
  cudaFree(p->idx_d);
  cudaFree(p->inv_off_d);
  cudaFree(p->inv_ent_d);
  cudaFree(p->scratch_d);
  cudaFree(p->upd_d);
  delete p;
  return HASTE_OK;
}

haste_status_t haste_plan_info(haste_plan_t p, int64_t* index_bytes, int64_t* inverse_bytes) {
  if (!p) return fail(HASTE_ERR_INVALID_ARG, "plan is NULL");
  if (index_bytes) *index_bytes = 4 * p->n_groups * p->k;
  if (inverse_bytes) *inverse_bytes = 4 * ((int64_t)p->d + 1 + p->n_groups * p->k);
  return HASTE_OK;
}

haste_status_t haste_plan_export(haste_plan_t p, int32_t* idx, int32_t* inv_off, int32_t* inv_ent) {
  if (haste_status_t st = check_plan_device(p)) return st;
  const size_t n = (size_t)p->n_groups * p->k;
  if (idx) HASTE_CUDA(cudaMemcpy(idx, p->idx_d, n * 4, cudaMemcpyDeviceToHost));
  if (inv_off) HASTE_CUDA(cudaMemcpy(inv_off, p->inv_off_d, ((size_t)p->d + 1) * 4, cudaMemcpyDeviceToHost));
  if (inv_ent) HASTE_CUDA(cudaMemcpy(inv_ent, p->inv_ent_d, n * 4, cudaMemcpyDeviceToHost));
  return HASTE_OK;
}

size_t haste_workspace_size(haste_plan_t p, int32_t B, haste_dtype_t dt) {
  if (!p || B <= 0 || check_plan_device(p) != HASTE_OK) return 0;
  DeviceInfo di;
  if (device_info(di) != HASTE_OK) return 0;
  const int Bp = round_up(B, 128);
  const DxTiling t = dx_tiling(*p, Bp, elem_bytes(dt), di.sms, di.smem_optin);
  return tail_ws(*p, B, elem_bytes(dt), t).total;
}

haste_status_t haste_forward(haste_plan_t p, int32_t B, haste_dtype_t dt, const void* X, const void* W,
                             void* logits, void* ws, size_t ws_bytes, haste_stream_t stream) {
  DeviceInfo di;
  haste_status_t st = device_info(di);
  if (st == HASTE_OK) st = check_tail(p, B, dt, di);
  if (st != HASTE_OK) return st;
  if (!X || !W || !logits) return fail(HASTE_ERR_INVALID_ARG, "NULL tensor pointer");
  const int E = elem_bytes(dt);
  const DxTiling t = dx_tiling(*p, round_up(B, 128), E, di.sms, di.smem_optin);
  const TailWs w = tail_ws(*p, B, E, t);
  if ((st = check_ws(ws, ws_bytes, w.total)) != HASTE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  TailArgs a = make_args(*p, B);
  a.Xt = static_cast<uint8_t*>(ws) + w.xt;
  a.W = W;
  a.logits = logits;
  cudaError_t e;
  {
    ProfScope ps("xt", s);
    e = dt == HASTE_BF16 ? xt<__nv_bfloat16>(a, X, const_cast<void*>(a.Xt), s)
                         : xt<float>(a, X, const_cast<void*>(a.Xt), s);
  }
  if (e == cudaSuccess) {
    ProfScope ps("tail_forward", s);
    const int Bp = a.sh.Bp, ns = tail3::stages(p->k, p->G, (size_t)di.smem_optin, 4096, true);
    if (dt == HASTE_BF16 && tail3::supported(p->G, p->k, Bp) && ns > 0) {
      v3::GivenArgs g{};
      g.sh = a.sh;
      g.idx = p->idx_d;
      g.Xt = static_cast<const __nv_bfloat16*>(a.Xt);
      g.W = static_cast<const __nv_bfloat16*>(W);
      g.out = static_cast<__nv_bfloat16*>(logits);
      g.n_chunks = (int)std::min<int64_t>(p->n_groups, std::max(1, di.sms / (Bp / 128)));
      g.ns = ns;
      e = tail3::launch_fwd(p->G, p->k, g, s);
    } else {
      e = dt == HASTE_BF16 ? tail::launch_forward<__nv_bfloat16>(a, di.sms, s)
                           : tail::launch_forward<float>(a, di.sms, s);
    }
  }
  return e == cudaSuccess ? HASTE_OK : cuda_fail(e, "haste_forward launch");
}

haste_status_t haste_backward_dw(haste_plan_t p, int32_t B, haste_dtype_t dt, const void* X, const void* dY,
                                 void* dW, void* ws, size_t ws_bytes, haste_stream_t stream) {
  DeviceInfo di;
  haste_status_t st = device_info(di);
  if (st == HASTE_OK) st = check_tail(p, B, dt, di);
  if (st != HASTE_OK) return st;
  if (!X || !dY || !dW) return fail(HASTE_ERR_INVALID_ARG, "NULL tensor pointer");
  const int E = elem_bytes(dt);
  const DxTiling t = dx_tiling(*p, round_up(B, 128), E, di.sms, di.smem_optin);
  const TailWs w = tail_ws(*p, B, E, t);
  if ((st = check_ws(ws, ws_bytes, w.total)) != HASTE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  TailArgs a = make_args(*p, B);
  a.Xt = static_cast<uint8_t*>(ws) + w.xt;
  a.dY = dY;
  a.dW = dW;
  cudaError_t e;
  {
    ProfScope ps("xt", s);
    e = dt == HASTE_BF16 ? xt<__nv_bfloat16>(a, X, const_cast<void*>(a.Xt), s)
                         : xt<float>(a, X, const_cast<void*>(a.Xt), s);
  }
  if (e == cudaSuccess) {
    ProfScope ps("tail_dw", s);
    const int Bp = a.sh.Bp, ns = tail3::stages(p->k, p->G, (size_t)di.smem_optin, 4096, false);
    if (dt == HASTE_BF16 && tail3::supported(p->G, p->k, Bp) && ns > 0) {
      v3::GivenArgs g{};
      g.sh = a.sh;
      g.idx = p->idx_d;
      g.Xt = static_cast<const __nv_bfloat16*>(a.Xt);
      g.dY = static_cast<const __nv_bfloat16*>(dY);
      g.out = static_cast<__nv_bfloat16*>(dW);
      g.n_chunks = (int)std::min<int64_t>(p->n_groups, di.sms);
      g.ns = ns;
      e = tail3::launch_dw(p->G, p->k, g, s);
    } else {
      e = dt == HASTE_BF16 ? tail::launch_backward_dw<__nv_bfloat16>(a, di.sms, s)
                           : tail::launch_backward_dw<float>(a, di.sms, s);
    }
  }
  return e == cudaSuccess ? HASTE_OK : cuda_fail(e, "haste_backward_dw launch");
}

haste_status_t haste_backward_dx(haste_plan_t p, int32_t B, haste_dtype_t dt, const void* W, const void* dY,
                                 float* dX, int accumulate, void* ws, size_t ws_bytes, haste_stream_t stream) {
  DeviceInfo di;
  haste_status_t st = device_info(di);
  if (st == HASTE_OK) st = check_tail(p, B, dt, di);
  if (st != HASTE_OK) return st;
  if (!W || !dY || !dX) return fail(HASTE_ERR_INVALID_ARG, "NULL tensor pointer");
  const int E = elem_bytes(dt);
  const DxTiling t = dx_tiling(*p, round_up(B, 128), E, di.sms, di.smem_optin);
  const TailWs w = tail_ws(*p, B, E, t);
  if ((st = check_ws(ws, ws_bytes, w.total)) != HASTE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  TailArgs a = make_args(*p, B);
  a.W = W;
  a.dY = dY;
  a.dX_part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w.dx_part);
  a.band = t.band;
  a.n_bands = t.n_bands;
  a.n_chunks = t.n_chunks;
  cudaError_t e;
  {
    ProfScope ps("tail_dx", s);
    if (t.ns > 0)
      e = dx_v2(*p, B, W, dY, false, a.dX_part, t, s);
    else
      e = dt == HASTE_BF16 ? tail::launch_backward_dx<__nv_bfloat16>(a, false, s)
                           : tail::launch_backward_dx<float>(a, false, s);
  }
  if (e == cudaSuccess) {
    ProfScope ps("dx_reduce", s);
    e = tail::launch_dx_reduce(a.dX_part, dX, t.n_chunks, p->d, a.sh.Bp, B, accumulate, s);
  }
  return e == cudaSuccess ? HASTE_OK : cuda_fail(e, "haste_backward_dx launch");
}

// dX without a workspace and without any allocation: the chunk partials live in
// the library's static scratch (16 MiB), so the group chunks of the reduction
// are capped to what fits there.  Same result definition as haste_backward_dx;
// the cap can change the chunking and hence the rounding of the chunk sums.
haste_status_t haste_backward_dx_noalloc(haste_plan_t p, int32_t B, haste_dtype_t dt, const void* W, const void* dY,
                                         float* dX, int accumulate, haste_stream_t stream) {
  DeviceInfo di;
  haste_status_t st = device_info(di);
  if (st == HASTE_OK) st = check_tail(p, B, dt, di);
  if (st != HASTE_OK) return st;
  if (!W || !dY || !dX) return fail(HASTE_ERR_INVALID_ARG, "NULL tensor pointer");
  const int E = elem_bytes(dt);
  const int Bp = round_up(B, 128);
  DxTiling t = dx_tiling(*p, Bp, E, di.sms, di.smem_optin);
  const size_t per_chunk = (size_t)p->d * Bp * 4;
  const size_t max_chunks = kNoAllocScratchBytes / per_chunk;
  if (max_chunks < 1)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE,
                "haste_backward_dx_noalloc needs d*roundup(B,128)*4 = %zu bytes of scratch; its static scratch "
                "holds %zu bytes",
                per_chunk, kNoAllocScratchBytes);
  if ((size_t)t.n_chunks > max_chunks) t.n_chunks = (int)max_chunks;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != HASTE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  TailArgs a = make_args(*p, B);
  a.W = W;
  a.dY = dY;
  a.dX_part = static_cast<float*>(scratch);
  a.band = t.band;
  a.n_bands = t.n_bands;
  a.n_chunks = t.n_chunks;
  cudaError_t e = t.ns > 0 ? dx_v2(*p, B, W, dY, false, a.dX_part, t, s)
                 : dt == HASTE_BF16  ? tail::launch_backward_dx<__nv_bfloat16>(a, false, s)
                                     : tail::launch_backward_dx<float>(a, false, s);
  if (e == cudaSuccess) e = tail::launch_dx_reduce(a.dX_part, dX, t.n_chunks, p->d, Bp, B, accumulate, s);
  return e == cudaSuccess ? HASTE_OK : cuda_fail(e, "haste_backward_dx_noalloc launch");
}

}  // extern "C"

namespace {

// Optimizer update fused into the step kernel's dW readout (haste_bce_step_sgd).
struct SgdUpdate {
  float lr, momentum;
  void* M;      // momentum [L, k] in W's dtype, NULL when momentum == 0
  void* W_out;  // updated weights [L, k]
};

haste_status_t bce_step_impl(haste_plan_t p, int32_t B, haste_dtype_t dt, const void* X, const void* W,
                             haste_targets_t pos, float grad_scale, float* loss, void* dW, const SgdUpdate* upd,
                             float* dX, int accumulate, void* ws, size_t ws_bytes, haste_stream_t stream) {
  DeviceInfo di;
  haste_status_t st = device_info(di);
  if (st == HASTE_OK) st = check_tail(p, B, dt, di);
  if (st != HASTE_OK) return st;
  if (!X || !W || (!upd && !dW) || !dX || !pos.row_ptr || !pos.ids) return fail(HASTE_ERR_INVALID_ARG, "NULL pointer");
  const int E = elem_bytes(dt);
  const int Bp = round_up(B, 128);
  if ((Bp / 128) * p->G + (E == 4 ? (p->G + 31) / 32 * 32 : p->G) > 512)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "(B/128 + 1) * G must fit the 512 TMEM columns");
  if (tail::smem_step(E, p->k, p->G, Bp) > (size_t)di.smem_optin)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "fused step tiles exceed shared memory");
  const DxTiling t = dx_tiling(*p, Bp, E, di.sms, di.smem_optin);
  const TailWs w = tail_ws(*p, B, E, t);
  if ((st = check_ws(ws, ws_bytes, w.total)) != HASTE_OK) return st;
  const bool v2p = use_v2(*p, Bp, E) && tail2::step_smem(Bp, p->k, p->G) <= (size_t)di.smem_optin && t.ns > 0;
  if (upd && !v2p)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE,
                "the fused update needs bf16, G in {16,32,64}, k in {64,128} and B <= 256");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  TailArgs a = make_args(*p, B);
  a.Xt = wb + w.xt;
  a.W = W;
  a.dW = dW;
  a.dY_out = wb + w.dy_buf;
  a.dX_part = reinterpret_cast<float*>(wb + w.dx_part);
  a.loss_part = reinterpret_cast<float*>(wb + w.loss_part);
  a.pos_ptr = pos.row_ptr;
  a.pos_ids = pos.ids;
  a.grad_scale = grad_scale;
  a.band = t.band;
  a.n_bands = t.n_bands;
  a.n_chunks = t.n_chunks;
  const int grid = v2p ? (int)std::min<int64_t>(p->n_groups, di.sms)
                       : dt == HASTE_BF16 ? tail::step_grid<__nv_bfloat16>(a, di.sms) : tail::step_grid<float>(a, di.sms);
  if (grid <= 0 || grid > kMaxLossParts) return fail(HASTE_ERR_CUDA, "could not size the fused step grid");
  cudaError_t e;
  {
    ProfScope ps("xt", s);
    e = dt == HASTE_BF16 ? xt<__nv_bfloat16>(a, X, const_cast<void*>(a.Xt), s)
                         : xt<float>(a, X, const_cast<void*>(a.Xt), s);
  }
  if (e == cudaSuccess) {
    ProfScope ps("tail_step", s);
    if (v2p) {
      v2::StepArgs sa{};
      sa.sh = a.sh;
      sa.idx = p->idx_d;
      sa.dW = static_cast<__nv_bfloat16*>(dW);
      auto a32 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 31) == 0; };
      sa.out_v8 = a32(dW);
      sa.dY_out = static_cast<__nv_bfloat16*>(a.dY_out);
      sa.loss_part = a.loss_part;
      sa.pos_ptr = pos.row_ptr;
      sa.pos_ids = pos.ids;
      sa.grad_scale = grad_scale;
      int mode = 0;
      if (upd) {
        sa.W_out = static_cast<__nv_bfloat16*>(upd->W_out);
        sa.M = static_cast<__nv_bfloat16*>(upd->M);
        sa.lr = upd->lr;
        sa.momentum = upd->momentum;
        mode = upd->momentum != 0.f ? 2 : 1;
        sa.out_v8 = a32(upd->W_out) && (mode == 1 || a32(upd->M));
      }
      e = tail2::launch_step(p->G, p->k, mode, sa, grid, a.Xt, W, s);
    } else {
      e = dt == HASTE_BF16 ? tail::launch_step<__nv_bfloat16>(a, grid, s) : tail::launch_step<float>(a, grid, s);
    }
  }
  if (e == cudaSuccess) {
    ProfScope ps("tail_dx", s);
    if (v2p)
      e = dx_v2(*p, B, W, a.dY_out, true, a.dX_part, t, s);
    else if (t.ns > 0)
      e = dx_v2(*p, B, W, a.dY_out, false, a.dX_part, t, s);
    else
      e = dt == HASTE_BF16 ? tail::launch_backward_dx<__nv_bfloat16>(a, true, s)
                           : tail::launch_backward_dx<float>(a, true, s);
  }
  if (e == cudaSuccess) {  // the chunk partials of dX and, with a loss pointer, the loss partials
    ProfScope ps("dx_reduce", s);
    e = tail::launch_dx_reduce(a.dX_part, dX, t.n_chunks, p->d, Bp, B, accumulate, s, loss ? a.loss_part : nullptr,
                               grid, grad_scale, loss);
  }
  return e == cudaSuccess ? HASTE_OK : cuda_fail(e, upd ? "haste_bce_step_sgd launch" : "haste_bce_step launch");
}

}  // namespace

extern "C" {

haste_status_t haste_bce_step(haste_plan_t p, int32_t B, haste_dtype_t dt, const void* X, const void* W,
                              haste_targets_t pos, float grad_scale, float* loss, void* dW, float* dX,
                              int accumulate, void* ws, size_t ws_bytes, haste_stream_t stream) {
  return bce_step_impl(p, B, dt, X, W, pos, grad_scale, loss, dW, nullptr, dX, accumulate, ws, ws_bytes, stream);
}

haste_status_t haste_bce_step_sgd(haste_plan_t p, int32_t B, haste_dtype_t dt, const void* X, const void* W,
                                  haste_targets_t pos, float grad_scale, float* loss, float lr, float momentum,
                                  void* M, void* W_out, float* dX, int accumulate, void* ws, size_t ws_bytes,
                                  haste_stream_t stream) {
  if (!W_out) return fail(HASTE_ERR_INVALID_ARG, "W_out is NULL");
  if (W_out == W) return fail(HASTE_ERR_INVALID_ARG, "W_out must not be W: the dX pass reads W after the update");
  if (momentum != 0.f && !M) return fail(HASTE_ERR_INVALID_ARG, "momentum != 0 needs the momentum buffer M");
  if (M && (M == W || M == W_out)) return fail(HASTE_ERR_INVALID_ARG, "M must be its own buffer");
  if (!(lr == lr) || !(momentum == momentum)) return fail(HASTE_ERR_INVALID_ARG, "lr and momentum must be numbers");
  const SgdUpdate u{lr, momentum, momentum != 0.f ? M : nullptr, W_out};
  return bce_step_impl(p, B, dt, X, W, pos, grad_scale, loss, nullptr, &u, dX, accumulate, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------- head
namespace {
struct HeadWs {
  size_t loss_part, dxh_part, total;
};
HeadWs head_ws(int B, int H, int d, int E) {
  HeadWs w{};
  size_t off = 0;
  w.loss_part = off;
  off = align256(off + (size_t)head::fwd_tiles(B, H) * 4);
  w.dxh_part = off;
  const int S = head::dxh_splits(H, E);
  off = align256(off + (S > 1 ? (size_t)S * B * d * 4 : 0));
  w.total = off;
  return w;
}
haste_status_t check_head(int B, int H, int d, haste_dtype_t dt) {
  if (dt != HASTE_F32 && dt != HASTE_BF16) return fail(HASTE_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  if (B <= 0 || H <= 0 || d <= 0) return fail(HASTE_ERR_INVALID_ARG, "B, H and d must be positive");
  const int E = elem_bytes(dt);
  if ((d * E) % 16 || (H * E) % 16)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "H and d must be multiples of %d", 16 / E);
  return HASTE_OK;
}
}  // namespace

// Workspace of haste_topk: X^T [d, Bp] (input dtype) and the stage-1 candidates
// [n_buckets][Bp][kp] (fp32 values, int32 label ids).
static size_t topk_ws(const haste_plan_s& p, int B, int E, int n_buckets, int kp, size_t* cand) {
  const int Bp = round_up(B, 128);
  *cand = align256((size_t)p.d * Bp * E);
  return *cand + align256((size_t)n_buckets * Bp * kp * 8);
}

size_t haste_topk_workspace_size(haste_plan_t p, int32_t B, haste_dtype_t dt, int32_t n_buckets, int32_t kp) {
  if (!p || B <= 0 || n_buckets <= 0 || kp <= 0 || check_plan_device(p) != HASTE_OK) return 0;
  size_t cand;
  return topk_ws(*p, B, elem_bytes(dt), n_buckets, kp, &cand);
}

haste_status_t haste_topk(haste_plan_t p, int32_t B, haste_dtype_t dt, const void* X, const void* W, int32_t k,
                          int32_t kp, int32_t n_buckets, float* out_val, int32_t* out_id, void* ws, size_t ws_bytes,
                          haste_stream_t stream) {
  DeviceInfo di;
  haste_status_t st = device_info(di);
  if (st == HASTE_OK) st = check_tail(p, B, dt, di);
  if (st != HASTE_OK) return st;
  if (!X || !W || !out_val || !out_id) return fail(HASTE_ERR_INVALID_ARG, "NULL pointer");
  const int Bp = round_up(B, 128);
  if (dt != HASTE_BF16 || !topk_host::supported(p->G, p->k, Bp, kp))
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE,
                "top-k scoring needs bf16, G in {16,32,64}, k in {64,128}, B <= 256, kp in {1,2,4,8}");
  if (n_buckets < 1 || (int64_t)n_buckets > p->n_groups)
    return fail(HASTE_ERR_INVALID_ARG, "n_buckets=%d must lie in [1, n_groups]", n_buckets);
  if (k < 1 || k > 64 || (int64_t)k > (int64_t)n_buckets * kp)
    return fail(HASTE_ERR_INVALID_ARG, "k=%d must lie in [1, min(64, n_buckets * kp)]", k);
  if ((size_t)n_buckets * kp * 8 > (size_t)di.smem_optin - 1024)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "n_buckets * kp candidates exceed shared memory");
  if (topk_host::smem_stage1(Bp, p->k, p->G, kp) > (size_t)di.smem_optin)
    return fail(HASTE_ERR_UNSUPPORTED_SHAPE, "top-k tiles exceed shared memory");
  size_t cand;
  const size_t need = topk_ws(*p, B, 2, n_buckets, kp, &cand);
  if ((st = check_ws(ws, ws_bytes, need)) != HASTE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  TailArgs xa = make_args(*p, B);
  xa.Xt = wb;
  topk::Args a{};
  a.sh = xa.sh;
  a.idx = p->idx_d;
  a.cand_val = reinterpret_cast<float*>(wb + cand);
  a.cand_id = reinterpret_cast<int32_t*>(wb + cand + (size_t)n_buckets * Bp * kp * 4);
  cudaError_t e;
  {
    ProfScope ps("xt", s);
    e = xt<__nv_bfloat16>(xa, X, wb, s);
  }
  if (e == cudaSuccess) {
    ProfScope ps("topk_score", s);
    e = topk_host::launch_stage1(p->G, p->k, kp, a, n_buckets, wb, W, s);
  }
  if (e == cudaSuccess) {
    ProfScope ps("topk_merge", s);
    e = topk_host::launch_stage2(a.cand_val, a.cand_id, B, Bp, n_buckets, kp, k, out_val, out_id, s);
  }
  return e == cudaSuccess ? HASTE_OK : cuda_fail(e, "haste_topk launch");
}

size_t haste_head_workspace_size(int32_t B, int32_t H, int32_t d, haste_dtype_t dt) {
  if (B <= 0 || H <= 0 || d <= 0) return 0;
  return head_ws(B, H, d, elem_bytes(dt)).total;
}

haste_status_t haste_head_forward(int32_t B, int32_t H, int32_t d, haste_dtype_t dt, const void* Xh, const void* Wh,
                                  void* out, const haste_targets_t* pos, float grad_scale, float* loss, void* ws,
                                  size_t ws_bytes, haste_stream_t stream) {
  DeviceInfo di;
  haste_status_t st = device_info(di);
  if (st == HASTE_OK) st = check_head(B, H, d, dt);
  if (st != HASTE_OK) return st;
  if (!Xh || !Wh || !out) return fail(HASTE_ERR_INVALID_ARG, "NULL tensor pointer");
  if (pos && (!pos->row_ptr || !pos->ids)) return fail(HASTE_ERR_INVALID_ARG, "NULL targets");
  const HeadWs w = head_ws(B, H, d, elem_bytes(dt));
  if ((st = check_ws(ws, ws_bytes, w.total)) != HASTE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* lp = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w.loss_part);
  const int32_t* rp = pos ? pos->row_ptr : nullptr;
  const int32_t* ids = pos ? pos->ids : nullptr;
  cudaError_t e;
  {
    ProfScope ps("head_forward", s);
    e = dt == HASTE_BF16 ? head::forward<__nv_bfloat16>(B, H, d, Xh, Wh, out, rp, ids, grad_scale, lp, s)
                         : head::forward<float>(B, H, d, Xh, Wh, out, rp, ids, grad_scale, lp, s);
  }
  if (e == cudaSuccess && pos && loss) {
    ProfScope ps("loss_reduce", s);
    e = tail::launch_loss_reduce(lp, head::fwd_tiles(B, H), grad_scale, loss, s);
  }
  return e == cudaSuccess ? HASTE_OK : cuda_fail(e, "haste_head_forward launch");
}

haste_status_t haste_head_backward(int32_t B, int32_t H, int32_t d, haste_dtype_t dt, const void* Xh, const void* Wh,
                                   const void* dYh, void* dWh, float* dXh, void* ws, size_t ws_bytes,
                                   haste_stream_t stream) {
  DeviceInfo di;
  haste_status_t st = device_info(di);
  if (st == HASTE_OK) st = check_head(B, H, d, dt);
  if (st != HASTE_OK) return st;
  if (!Xh || !Wh || !dYh || !dWh || !dXh) return fail(HASTE_ERR_INVALID_ARG, "NULL tensor pointer");
  const HeadWs w = head_ws(B, H, d, elem_bytes(dt));
  if ((st = check_ws(ws, ws_bytes, w.total)) != HASTE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w.dxh_part);
  cudaError_t e;
  {
    ProfScope ps("head_dw", s);
    e = dt == HASTE_BF16 ? head::backward_dw<__nv_bfloat16>(B, H, d, Xh, dYh, dWh, s)
                         : head::backward_dw<float>(B, H, d, Xh, dYh, dWh, s);
  }
  if (e == cudaSuccess) {
    ProfScope ps("head_dx", s);
    e = dt == HASTE_BF16 ? head::backward_dx<__nv_bfloat16>(B, H, d, Wh, dYh, dXh, part, s)
                         : head::backward_dx<float>(B, H, d, Wh, dYh, dXh, part, s);
  }
  return e == cudaSuccess ? HASTE_OK : cuda_fail(e, "haste_head_backward launch");
}

}  // extern "C"
