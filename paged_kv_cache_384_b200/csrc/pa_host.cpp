// pa_host.cpp -- host runtime of libpagedattn: error reporting, device queries, the
// device error word, profiling hooks, the block manager and the slot-mapping helper.
#include "pa_host.h"

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

namespace pa {

namespace {
thread_local std::string t_last_error;

std::mutex& registry_mutex() {
  static std::mutex m;
  return m;
}
std::vector<DeviceErrorReader>& readers() {
  static std::vector<DeviceErrorReader> r;
  return r;
}
}  // namespace

pa_status fail(pa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

pa_status cuda_fail(cudaError_t err, const char* what) {
  return fail(PA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(err), cudaGetErrorName(err));
}

pa_status current_device(int* device, int* sm_count) {
  static int cached[256] = {0};
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 256) return fail(PA_ERR_CUDA, "device ordinal %d out of range", dev);
  if (cached[dev] == 0) {
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(MultiProcessorCount)");
    cached[dev] = n;
  }
  *device = dev;
  *sm_count = cached[dev];
  return PA_OK;
}

cudaError_t launch_dependent(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

void register_device_error_reader(DeviceErrorReader reader) {
  std::lock_guard<std::mutex> lock(registry_mutex());
  readers().push_back(reader);
}

// ---------------------------------------------------------------------------------------
// Profiling: a growing pool of event triplets, recorded by the decode entry point.
// ---------------------------------------------------------------------------------------
namespace {
struct Profiler {
  std::mutex m;
  bool on = false;
  std::vector<cudaEvent_t> events;  // 3 per call
  size_t used = 0;                  // calls recorded since reset
};
Profiler& profiler() {
  static Profiler p;
  return p;
}
}  // namespace

bool profiling_enabled() { return profiler().on; }

void profiling_next_events(cudaEvent_t* ev) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> lock(p.m);
  ev[0] = ev[1] = ev[2] = nullptr;
  if (!p.on) return;
  const size_t need = 3 * (p.used + 1);
  while (p.events.size() < need) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    p.events.push_back(e);
  }
  for (int i = 0; i < 3; ++i) ev[i] = p.events[3 * p.used + i];
  ++p.used;
}

}  // namespace pa

using namespace pa;

extern "C" {

const char* pa_last_error(void) { return t_last_error.c_str(); }

const char* pa_version(void) { return "pagedattn 0.1.0 (sm_100a)"; }

pa_status pa_device_error(uint32_t* flags, int clear) {
  if (!flags) return fail(PA_ERR_INVALID_ARG, "pa_device_error: flags is NULL");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  uint32_t all = 0;
  std::vector<DeviceErrorReader> rs;
  {
    std::lock_guard<std::mutex> lock(registry_mutex());
    rs = readers();
  }
  for (DeviceErrorReader r : rs) {
    uint32_t f = 0;
    e = r(&f, clear);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    all |= f;
  }
  *flags = all;
  return PA_OK;
}

pa_status pa_profile_enable(int on) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> lock(p.m);
  p.on = on != 0;
  return PA_OK;
}

pa_status pa_profile_read(double* partition_ms, double* merge_ms, int* calls, int reset) {
  Profiler& p = profiler();
  std::lock_guard<std::mutex> lock(p.m);
  double a = 0.0, b = 0.0;
  for (size_t i = 0; i < p.used; ++i) {
    cudaEvent_t* ev = &p.events[3 * i];
    cudaError_t e = cudaEventSynchronize(ev[2]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    float x = 0.f, y = 0.f;
    e = cudaEventElapsedTime(&x, ev[0], ev[1]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    e = cudaEventElapsedTime(&y, ev[1], ev[2]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    a += x;
    b += y;
  }
  if (partition_ms) *partition_ms = a;
  if (merge_ms) *merge_ms = b;
  if (calls) *calls = static_cast<int>(p.used);
  if (reset) p.used = 0;
  return PA_OK;
}

// ---------------------------------------------------------------------------------------
// Block manager: free list (popped from its end) + reference counts.
// ---------------------------------------------------------------------------------------
struct pa_block_manager {
  int num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_list;
  std::vector<int32_t> ref_count;
};

pa_block_manager* pa_bm_create(int num_blocks, int block_size, const int32_t* free_order) {
  if (num_blocks <= 0 || block_size <= 0) {
    fail(PA_ERR_INVALID_ARG, "pa_bm_create: num_blocks and block_size must be positive");
    return nullptr;
  }
  auto* bm = new pa_block_manager;
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->ref_count.assign(num_blocks, 0);
  bm->free_list.resize(num_blocks);
  if (free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        fail(PA_ERR_INVALID_ARG, "pa_bm_create: free_order is not a permutation of 0..%d",
             num_blocks - 1);
        return nullptr;
      }
      seen[b] = 1;
      bm->free_list[i] = b;
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) bm->free_list[i] = i;
  }
  return bm;
}

void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

pa_status pa_bm_allocate(pa_block_manager* bm, int n, int32_t* out_ids) {
  if (!bm || n < 0 || (n > 0 && !out_ids)) return fail(PA_ERR_INVALID_ARG, "pa_bm_allocate: bad argument");
  if (static_cast<size_t>(n) > bm->free_list.size())
    return fail(PA_ERR_OUT_OF_BLOCKS, "out of blocks: need %d, %zu free", n, bm->free_list.size());
  for (int i = 0; i < n; ++i) {
    const int32_t b = bm->free_list.back();
    bm->free_list.pop_back();
    bm->ref_count[b] = 1;
    out_ids[i] = b;
  }
  return PA_OK;
}

pa_status pa_bm_free(pa_block_manager* bm, const int32_t* ids, int n) {
  if (!bm || n < 0 || (n > 0 && !ids)) return fail(PA_ERR_INVALID_ARG, "pa_bm_free: bad argument");
  // Validate the whole request first (a block may appear several times).
  std::unordered_map<int32_t, int> need;
  for (int i = 0; i < n; ++i) {
    const int32_t b = ids[i];
    if (b < 0 || b >= bm->num_blocks) return fail(PA_ERR_BAD_BLOCK, "free: block %d out of range", b);
    if (++need[b] > bm->ref_count[b])
      return fail(PA_ERR_BAD_BLOCK, "free: block %d reference count would go negative (double free)", b);
  }
  for (int i = 0; i < n; ++i) {
    const int32_t b = ids[i];
    if (--bm->ref_count[b] == 0) bm->free_list.push_back(b);
  }
  return PA_OK;
}

pa_status pa_bm_share(pa_block_manager* bm, const int32_t* ids, int n) {
  if (!bm || n < 0 || (n > 0 && !ids)) return fail(PA_ERR_INVALID_ARG, "pa_bm_share: bad argument");
  for (int i = 0; i < n; ++i) {
    const int32_t b = ids[i];
    if (b < 0 || b >= bm->num_blocks || bm->ref_count[b] <= 0)
      return fail(PA_ERR_BAD_BLOCK, "share: block %d is not allocated", b);
  }
  for (int i = 0; i < n; ++i) ++bm->ref_count[ids[i]];
  return PA_OK;
}

pa_status pa_bm_copy_on_write(pa_block_manager* bm, int32_t block_id, int32_t* out_id) {
  if (!bm || !out_id) return fail(PA_ERR_INVALID_ARG, "pa_bm_copy_on_write: bad argument");
  if (block_id < 0 || block_id >= bm->num_blocks)
    return fail(PA_ERR_BAD_BLOCK, "copy_on_write: block %d out of range", block_id);
  if (bm->ref_count[block_id] <= 1) {
    *out_id = block_id;
    return PA_OK;
  }
  int32_t fresh = -1;
  pa_status st = pa_bm_allocate(bm, 1, &fresh);
  if (st != PA_OK) return st;
  --bm->ref_count[block_id];
  *out_id = fresh;
  return PA_OK;
}

int pa_bm_num_free(const pa_block_manager* bm) { return bm ? static_cast<int>(bm->free_list.size()) : -1; }

int pa_bm_ref_count(const pa_block_manager* bm, int32_t block_id) {
  if (!bm || block_id < 0 || block_id >= bm->num_blocks) return -1;
  return bm->ref_count[block_id];
}

double pa_bm_usage_ratio(const pa_block_manager* bm) {
  if (!bm) return NAN;
  return 1.0 - static_cast<double>(bm->free_list.size()) / bm->num_blocks;
}

pa_status pa_bm_free_list(const pa_block_manager* bm, int32_t* out, int cap, int* n) {
  if (!bm || !n || cap < 0 || (cap > 0 && !out)) return fail(PA_ERR_INVALID_ARG, "pa_bm_free_list: bad argument");
  const int len = static_cast<int>(bm->free_list.size());
  *n = len;
  for (int i = 0; i < len && i < cap; ++i) out[i] = bm->free_list[i];
  return PA_OK;
}

pa_status pa_slot_mapping_host(const int32_t* block_tables, int num_seqs, int max_blocks_per_seq,
                               int block_size, const int32_t* seq, const int32_t* pos, int n,
                               int64_t* out) {
  if (n < 0 || (n > 0 && (!block_tables || !seq || !pos || !out)) || block_size <= 0 ||
      max_blocks_per_seq <= 0 || num_seqs < 0)
    return fail(PA_ERR_INVALID_ARG, "pa_slot_mapping_host: bad argument");
  for (int i = 0; i < n; ++i) {
    const int s = seq[i], p = pos[i];
    if (s < 0 || s >= num_seqs || p < 0 || p / block_size >= max_blocks_per_seq)
      return fail(PA_ERR_INVALID_ARG, "slot mapping: entry %d (seq %d, pos %d) outside the table", i, s, p);
    const int32_t pb = block_tables[static_cast<size_t>(s) * max_blocks_per_seq + p / block_size];
    if (pb < 0)
      return fail(PA_ERR_INVALID_ARG, "slot mapping: seq %d pos %d maps to unallocated block", s, p);
    out[i] = static_cast<int64_t>(pb) * block_size + p % block_size;
  }
  return PA_OK;
}

}  // extern "C"
