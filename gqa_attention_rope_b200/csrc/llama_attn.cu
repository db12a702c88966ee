// llama_attn.cu -- the library's single translation unit: host-side argument
// checks, TMA descriptor encoding, per-device caches (RoPE tables, scratch) and
// kernel launches behind the C ABI declared in include/llama_attn.h.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "llama_attn.h"
#include "ptx.cuh"
#include "rope.cuh"
#include "prefill_f32.cuh"
#include "prefill_bf16.cuh"
#include "qkv_fp8.cuh"
#include "decode.cuh"

#define LLAMA_ATTN_VERSION 300  // 0.3.0: caller-workspace prefill entry points, caller-owned RoPE table

namespace {

constexpr int kMaxDevices = 64;

struct RopeTable {
  double theta = 0.0;
  int D = 0;
  int maxpos = 0;
  float2* ptr = nullptr;
};

// Library-owned buffers behind the convenience entry points (the *_ws entry
// points take caller memory instead and touch none of these).
struct DeviceCache {
  std::vector<RopeTable> tables;
  void* prefill_ws = nullptr;  // rotated K, document starts, work-item counter
  size_t prefill_ws_bytes = 0;
  unsigned int* amax = nullptr;  // per-tensor amax of the E4M3 quantizer
  int32_t* doc_start = nullptr;  // document starts of the fp32 and FP8 paths
  size_t doc_bytes = 0;
};

// Per-device launch settings, set once (kernel attributes, SM count).
struct DeviceSetup {
  std::once_flag once;
  int status = 0;
  int n_sm = 148;
};

std::mutex g_mutex;
DeviceCache g_cache[kMaxDevices];
DeviceSetup g_setup[kMaxDevices];
std::atomic<unsigned int> g_epoch{0};

// Distinct, nonzero id per launch that uses bounded waits.
unsigned int next_epoch() {
  unsigned int e = ++g_epoch;
  if (e == 0) e = ++g_epoch;
  return e;
}

// ---- benchmark instrumentation (see llama_attn_profile_begin)
struct Profile {
  bool on = false;
  int device = -1;
  std::vector<cudaEvent_t> ev;  // pairs
  int pairs_used = 0;
  int launches = 0;
  int main_launches = 0;
};
Profile g_prof;
constexpr int kMaxProfiledPairs = 4096;

void prof_count(int n) {
  if (g_prof.on) g_prof.launches += n;
}
// Records the "before" event of a new pair; returns the pair index or -1.
int prof_before(cudaStream_t stream) {
  if (!g_prof.on) return -1;
  ++g_prof.main_launches;
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != g_prof.device || g_prof.pairs_used >= kMaxProfiledPairs) return -1;
  const int i = g_prof.pairs_used;
  if (static_cast<int>(g_prof.ev.size()) < 2 * (i + 1)) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess) return -1;
    if (cudaEventCreate(&b) != cudaSuccess) {
      cudaEventDestroy(a);
      return -1;
    }
    g_prof.ev.push_back(a);
    g_prof.ev.push_back(b);
  }
  if (cudaEventRecord(g_prof.ev[2 * i], stream) != cudaSuccess) return -1;
  g_prof.pairs_used = i + 1;
  return i;
}
void prof_after(int pair, cudaStream_t stream) {
  if (pair >= 0) cudaEventRecord(g_prof.ev[2 * pair + 1], stream);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? LLAMA_ATTN_OK : LLAMA_ATTN_ERR_CUDA; }

#define LA_CUDA(call)                                 \
  do {                                                \
    cudaError_t e_ = (call);                          \
    if (e_ != cudaSuccess) return LLAMA_ATTN_ERR_CUDA; \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return LLAMA_ATTN_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return LLAMA_ATTN_ERR_UNSUPPORTED;
  return LLAMA_ATTN_OK;
}

int grid_for(int64_t work, int threads) {
  int64_t blocks = (work + threads - 1) / threads;
  if (blocks > 148 * 32) blocks = 148 * 32;
  return static_cast<int>(blocks < 1 ? 1 : blocks);
}

// Cached cos/sin table with at least `maxpos` positions for (theta, D). The
// first build (or a growth) synchronises `stream` so later calls on any stream
// see a complete table.
int rope_table(DeviceCache& dc, double theta, int D, int maxpos, cudaStream_t stream, const float2** out) {
  for (auto& t : dc.tables) {
    if (t.theta == theta && t.D == D && t.maxpos >= maxpos) {
      *out = t.ptr;
      return LLAMA_ATTN_OK;
    }
  }
  RopeTable* slot = nullptr;
  for (auto& t : dc.tables)
    if (t.theta == theta && t.D == D) slot = &t;
  if (slot == nullptr) {
    dc.tables.push_back(RopeTable{});
    slot = &dc.tables.back();
  }
  if (slot->ptr) {
    LA_CUDA(cudaDeviceSynchronize());
    LA_CUDA(cudaFree(slot->ptr));
    slot->ptr = nullptr;
  }
  const int cap = maxpos < 4096 ? 4096 : maxpos;
  float2* ptr = nullptr;
  LA_CUDA(cudaMalloc(&ptr, sizeof(float2) * static_cast<size_t>(cap) * (D / 2)));
  slot->theta = theta;
  slot->D = D;
  slot->maxpos = cap;
  slot->ptr = ptr;
  prof_count(1);
  la::rope_table_kernel<<<grid_for(static_cast<int64_t>(cap) * (D / 2), 256), 256, 0, stream>>>(ptr, cap, D, theta);
  LA_CUDA(cudaGetLastError());
  LA_CUDA(cudaStreamSynchronize(stream));
  *out = ptr;
  return LLAMA_ATTN_OK;
}

int grow(void** buf, size_t* have, size_t need) {
  if (*have >= need) return LLAMA_ATTN_OK;
  if (*buf) {
    LA_CUDA(cudaDeviceSynchronize());
    LA_CUDA(cudaFree(*buf));
    *buf = nullptr;
    *have = 0;
  }
  LA_CUDA(cudaMalloc(buf, need));
  *have = need;
  return LLAMA_ATTN_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [B, S, H, 128] bf16 viewed as a 4-D tensor (d, h, s, b); box 64 x 1 x 128 x 1,
// 128-byte swizzle. Rows past S inside a batch row read as zero and are not
// written by stores.
int tmap_bshd(CUtensorMap* map, const void* ptr, int B, int S, int H) {
  auto enc = tensor_map_encoder();
  if (!enc) return LLAMA_ATTN_ERR_CUDA;
  const cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {256, static_cast<cuuint64_t>(H) * 256, static_cast<cuuint64_t>(S) * H * 256};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LLAMA_ATTN_OK : LLAMA_ATTN_ERR_CUDA;
}

// [rows, 128] bf16, box 64 x 64, 128-byte swizzle.
int tmap_rows(CUtensorMap* map, const void* ptr, int64_t rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return LLAMA_ATTN_ERR_CUDA;
  const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(la::dec::ROWS)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LLAMA_ATTN_OK : LLAMA_ATTN_ERR_CUDA;
}

// Row-major [rows, cols] matrix of 1- or 2-byte elements as a 2-D tensor map
// (cols innermost), box box_cols x box_rows, 128-byte swizzle (box_cols *
// elem_bytes == 128). Rows past `rows` read as zero and are not written.
int tmap_2d(CUtensorMap* map, const void* ptr, CUtensorMapDataType dt, int elem_bytes, int64_t rows, int64_t cols,
            int box_cols, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return LLAMA_ATTN_ERR_CUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem_bytes};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LLAMA_ATTN_OK : LLAMA_ATTN_ERR_CUDA;
}

int check_prefill_common(const void* q, const void* k, const void* v, const void* out, int B, int S, int Hq,
                         int Hkv, float rope_theta) {
  if (!q || !k || !v || !out) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * S > INT32_MAX - 1) return LLAMA_ATTN_ERR_UNSUPPORTED;
  return LLAMA_ATTN_OK;
}

// Once per device: the kernels' shared-memory attributes and the SM count.
// Thread-safe; no allocation, no synchronisation.
int device_setup(int dev, int* n_sm) {
  DeviceSetup& ds = g_setup[dev];
  std::call_once(ds.once, [&] {
    int st = LLAMA_ATTN_OK;
    auto attr = [&](const void* fn, uint32_t bytes) {
      if (st == LLAMA_ATTN_OK &&
          cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) != cudaSuccess)
        st = LLAMA_ATTN_ERR_CUDA;
    };
    attr(reinterpret_cast<const void*>(la::pfx::prefill_bf16_kernel), la::pfx::SMEM_ALLOC);
    attr(reinterpret_cast<const void*>(la::dec::decode_split_kernel<false>), la::dec::SMEM_ALLOC);
    attr(reinterpret_cast<const void*>(la::dec::decode_split_kernel<true>), la::dec::SMEM_ALLOC);
    attr(reinterpret_cast<const void*>(la::q8::qkv_fp8_rope_kernel), la::q8::SMEM_ALLOC);
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) ds.n_sm = n;
    ds.status = st;
  });
  if (n_sm) *n_sm = ds.n_sm;
  return ds.status;
}

}  // namespace

// ---- scratch for llama_attn_decode_noalloc
// A fixed device array replaces the caller's decode workspace for callers that
// cannot allocate device memory. Every device that loads this library holds it
// until the process exits. In host code the name is only a host-side handle:
// its device address comes from cudaGetSymbolAddress, once per device.
constexpr size_t kNoAllocScratchBytes = size_t(72) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
void* g_noalloc_scratch_addr[kMaxDevices];
}  // namespace

extern "C" {

int llama_attn_version(void) { return LLAMA_ATTN_VERSION; }

int llama_attn_profile_begin(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LLAMA_ATTN_ERR_CUDA;
  g_prof.on = true;
  g_prof.device = dev;
  g_prof.pairs_used = 0;
  g_prof.launches = 0;
  g_prof.main_launches = 0;
  return LLAMA_ATTN_OK;
}

int llama_attn_profile_end(double* main_kernel_ms, int* main_kernels_timed, int* kernels_launched) {
  std::lock_guard<std::mutex> lock(g_mutex);
  double total = 0.0;
  int st = LLAMA_ATTN_OK;
  for (int i = 0; i < g_prof.pairs_used; ++i) {
    float ms = 0.f;
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess) {
      st = LLAMA_ATTN_ERR_CUDA;
      break;
    }
    total += ms;
  }
  if (main_kernel_ms) *main_kernel_ms = total;
  if (main_kernels_timed) *main_kernels_timed = g_prof.pairs_used;
  if (kernels_launched) *kernels_launched = g_prof.launches;
  g_prof.on = false;
  return st;
}

const char* llama_attn_status_string(int status) {
  switch (status) {
    case LLAMA_ATTN_OK: return "ok";
    case LLAMA_ATTN_ERR_INVALID_ARG: return "invalid argument";
    case LLAMA_ATTN_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case LLAMA_ATTN_ERR_WORKSPACE: return "workspace or table missing, misaligned or too small";
    case LLAMA_ATTN_ERR_CUDA: return "CUDA runtime or launch failure";
    case LLAMA_ATTN_ERR_DEVICE: return "a kernel reported a device error";
    default: return "unknown status";
  }
}

int llama_attn_get_device_error(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return LLAMA_ATTN_ERR_CUDA;
  int err = 0;
  if (cudaMemcpyFromSymbol(&err, la::g_dev_error, sizeof(int)) != cudaSuccess) return LLAMA_ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(la::g_dev_error, &zero, sizeof(int)) != cudaSuccess) return LLAMA_ATTN_ERR_CUDA;
  return err;
}

}  // extern "C"

namespace {

// Query chunks (context parallelism): q holds S rows per batch row, rows
// [0, q_split) at global positions q_pos_a.., rows [q_split, S) at q_pos_b..;
// k and v hold the whole sequence, Skv rows. A plain prefill is
// Skv = q_split = S, q_pos_a = q_pos_b = 0.
struct QChunks {
  int Skv, q_split, q_pos_a, q_pos_b;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// The bf16 prefill's working memory, one block: the persistent kernel's
// work-item counter (256 B), per-token document starts (B*S int32) and the
// rotated keys (B*Skv*Hkv*128 bf16), each part 256-byte aligned.
struct PrefillWs {
  size_t doc_off, krot_off, total;
};
PrefillWs prefill_ws_layout(int64_t B, int64_t S, int64_t Hkv) {
  PrefillWs L;
  L.doc_off = 256;
  L.krot_off = L.doc_off + align256(static_cast<size_t>(B * S) * sizeof(int32_t));
  L.total = L.krot_off + align256(static_cast<size_t>(B * S * Hkv) * 128 * 2);
  return L;
}

// Everything the bf16 prefill launch needs besides the tensors: the RoPE
// table (rows = positions; may be null for pre-rotated inputs without a cache
// append) and the working memory laid out by prefill_ws_layout(B, max(S, Skv), Hkv).
struct PrefillRes {
  const float2* tab;
  int tab_rows;
  uint8_t* ws;
};

// The bf16 prefill: argument checks, then only kernel launches and a 4-byte
// memset on `stream` (no allocation, no synchronisation). lse, kcache and
// vcache may be null.
int prefill_bf16_launch(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                        llama_attn_bf16* out, float* lse, const int32_t* doc_offsets, int B, int S, int Hq, int Hkv,
                        llama_attn_bf16* kcache, llama_attn_bf16* vcache, int Lmax, const QChunks& qc,
                        bool prerotated, const PrefillRes& res, int dev, cudaStream_t stream) {
  const int Skv = qc.Skv;
  const int n_pos = S > Skv ? S : Skv;
  if (!prerotated || kcache) {
    if (res.tab == nullptr || res.tab_rows < n_pos) return LLAMA_ATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(res.tab) & 15u) return LLAMA_ATTN_ERR_INVALID_ARG;
  }
  int n_sm = 148, st;
  if ((st = device_setup(dev, &n_sm))) return st;
  const PrefillWs L = prefill_ws_layout(B, n_pos, Hkv);
  int* sched = reinterpret_cast<int*>(res.ws);
  int32_t* doc_start = doc_offsets ? reinterpret_cast<int32_t*>(res.ws + L.doc_off) : nullptr;
  void* krot = res.ws + L.krot_off;
  const int64_t ntok = static_cast<int64_t>(B) * S;
  const int64_t nkv_tok = static_cast<int64_t>(B) * Skv;
  const float4* tab4 = reinterpret_cast<const float4*>(res.tab);
  // The layout passes read the offsets once per block: one wave of blocks.
  auto stream_grid = [&](int64_t work) {
    const int g = grid_for(work, 256);
    return g < 8 * n_sm ? g : 8 * n_sm;
  };

  LA_CUDA(cudaMemsetAsync(sched, 0, sizeof(int), stream));
  const void* k_rot = k;  // pre-rotated keys are read as given
  if (!prerotated) {
    // K rotation; with document offsets it also writes the per-token starts
    const int64_t nvec_kv = nkv_tok * Hkv * 16;
    prof_count(1);
    la::rope_rotate_rows_bf16_kernel<<<stream_grid(nvec_kv), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(k), reinterpret_cast<uint4*>(krot), tab4, nullptr, doc_offsets, doc_start, B,
        Skv, Hkv, nvec_kv);
    LA_CUDA(cudaGetLastError());
    k_rot = krot;
  } else if (doc_offsets) {
    prof_count(1);
    la::doc_prep_kernel<<<stream_grid(ntok), 256, 0, stream>>>(doc_offsets, B, S, doc_start);
    LA_CUDA(cudaGetLastError());
  }
  if (kcache) {
    const int64_t nvec = ntok * Hkv * 16;
    prof_count(1);
    la::kv_cache_append_kernel<<<grid_for(nvec, 256), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v), tab4, doc_start,
        reinterpret_cast<uint4*>(kcache), reinterpret_cast<uint4*>(vcache), S, Hkv, Lmax, nvec);
    LA_CUDA(cudaGetLastError());
  }

  CUtensorMap tq, tk, tv, to;
  if ((st = tmap_bshd(&tq, q, B, S, Hq))) return st;
  if ((st = tmap_bshd(&tk, k_rot, B, Skv, Hkv))) return st;
  if ((st = tmap_bshd(&tv, v, B, Skv, Hkv))) return st;
  if ((st = tmap_bshd(&to, out, B, S, Hq))) return st;

  la::pfx::Params p;
  p.B = B;
  p.S = S;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.NH = (p.G % 2 == 0) ? 2 : 1;
  p.n_qt = (S + la::pfx::BM - 1) / la::pfx::BM;
  p.n_hp = Hq / p.NH;
  p.Skv = Skv;
  p.n_pos = n_pos;
  p.q_split = qc.q_split;
  p.q_pos_a = qc.q_pos_a;
  p.q_pos_b = qc.q_pos_b;
  p.q_rotated = prerotated ? 1 : 0;
  // Keys and values (rotated K and V) well beyond the 126 MB L2: run the items
  // KV group by KV group so the groups' tiles are read from DRAM about once.
  p.kv_major = (static_cast<int64_t>(B) * Skv * Hkv * 128 * 2 * 2 > (int64_t(256) << 20)) ? 1 : 0;
  p.doc_start = doc_start;
  p.rope_tab = tab4;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  p.epoch = next_epoch();
  p.sched = sched;
  p.lse = lse;
  const int64_t items = static_cast<int64_t>(B) * p.n_qt * p.n_hp;
  if (items > INT32_MAX) return LLAMA_ATTN_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(items < n_sm ? items : n_sm);
  prof_count(1);
  const int pair = prof_before(stream);
  la::pfx::prefill_bf16_kernel<<<grid, la::pfx::NTHREADS, la::pfx::SMEM_ALLOC, stream>>>(tq, tk, tv, to, p);
  const cudaError_t e = cudaGetLastError();
  prof_after(pair, stream);
  return cuda_status(e);
}

// Checks shared by every bf16 prefill entry point; done before any launch.
int check_prefill_bf16(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                       const llama_attn_bf16* out, const float* lse, int B, int S, int Hq, int Hkv, int D,
                       float rope_theta, const llama_attn_bf16* kcache, const llama_attn_bf16* vcache, int Lmax,
                       int Skv) {
  int st = check_prefill_common(q, k, v, out, B, S, Hq, Hkv, rope_theta);
  if (st) return st;
  if (Skv <= 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * Skv > INT32_MAX - 1) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (D != 128) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if ((kcache == nullptr) != (vcache == nullptr)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (kcache && (Lmax < S || !aligned16(kcache) || !aligned16(vcache))) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(S) * Hq * 256 >= (int64_t(1) << 40)) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(Skv) * Hkv * 256 >= (int64_t(1) << 40)) return LLAMA_ATTN_ERR_UNSUPPORTED;
  return LLAMA_ATTN_OK;
}

// Convenience form: the RoPE table and the working memory come from the
// library's per-device cache (allocated, or grown, on demand: that first use
// synchronises the device).
int prefill_bf16_cached(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                        llama_attn_bf16* out, float* lse, const int32_t* doc_offsets, int B, int S, int Hq, int Hkv,
                        int D, float rope_theta, llama_attn_bf16* kcache, llama_attn_bf16* vcache, int Lmax,
                        const QChunks& qc, cudaStream_t stream, bool prerotated = false) {
  int st = check_prefill_bf16(q, k, v, out, lse, B, S, Hq, Hkv, D, rope_theta, kcache, vcache, Lmax, qc.Skv);
  if (st) return st;
  int dev;
  if ((st = current_device(&dev))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCache& dc = g_cache[dev];
  const int n_pos = S > qc.Skv ? S : qc.Skv;
  PrefillRes res{nullptr, 0, nullptr};
  if (!prerotated || kcache) {
    if ((st = rope_table(dc, static_cast<double>(rope_theta), D, n_pos, stream, &res.tab))) return st;
    res.tab_rows = n_pos;
  }
  const size_t need = prefill_ws_layout(B, n_pos, Hkv).total;
  if ((st = grow(&dc.prefill_ws, &dc.prefill_ws_bytes, need))) return st;
  res.ws = static_cast<uint8_t*>(dc.prefill_ws);
  return prefill_bf16_launch(q, k, v, out, lse, doc_offsets, B, S, Hq, Hkv, kcache, vcache, Lmax, qc, prerotated,
                             res, dev, stream);
}

// Caller-memory form: nothing allocated, nothing synchronised.
int prefill_bf16_caller(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                        llama_attn_bf16* out, float* lse, const int32_t* doc_offsets, int B, int S, int Hq, int Hkv,
                        int D, const void* rope_table, int rope_rows, llama_attn_bf16* kcache,
                        llama_attn_bf16* vcache, int Lmax, const QChunks& qc, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  int st = check_prefill_bf16(q, k, v, out, lse, B, S, Hq, Hkv, D, 500000.f, kcache, vcache, Lmax, qc.Skv);
  if (st) return st;
  const int n_pos = S > qc.Skv ? S : qc.Skv;
  if (!rope_table || rope_rows < n_pos || (reinterpret_cast<uintptr_t>(rope_table) & 15u))
    return LLAMA_ATTN_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < prefill_ws_layout(B, n_pos, Hkv).total)
    return LLAMA_ATTN_ERR_WORKSPACE;
  int dev;
  if ((st = current_device(&dev))) return st;
  PrefillRes res{static_cast<const float2*>(rope_table), rope_rows, static_cast<uint8_t*>(workspace)};
  std::lock_guard<std::mutex> lock(g_mutex);  // only the benchmark instrumentation is shared
  return prefill_bf16_launch(q, k, v, out, lse, doc_offsets, B, S, Hq, Hkv, kcache, vcache, Lmax, qc, false, res,
                             dev, stream);
}

int check_cp(int B, int Sq, int Skv, int q_pos_a, int q_split, int q_pos_b) {
  if (B <= 0 || Sq <= 0 || Skv <= 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  constexpr int kT = la::pfx::BM;
  if (q_split < 0 || q_split > Sq || q_pos_a < 0 || q_pos_b < 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (q_split % kT != 0 || q_pos_a % kT != 0 || q_pos_b % kT != 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(q_pos_a) + q_split > Skv) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(q_pos_b) + (Sq - q_split) > Skv) return LLAMA_ATTN_ERR_INVALID_ARG;
  return LLAMA_ATTN_OK;
}

}  // namespace

extern "C" {

int llama_attn_prefill(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                       llama_attn_bf16* out, const int32_t* doc_offsets, int B, int S, int Hq, int Hkv, int D,
                       float rope_theta, cudaStream_t stream) {
  return prefill_bf16_cached(q, k, v, out, nullptr, doc_offsets, B, S, Hq, Hkv, D, rope_theta, nullptr, nullptr, 0,
                             QChunks{S, S, 0, 0}, stream);
}

int llama_attn_prefill_ex(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                          llama_attn_bf16* out, float* lse, const int32_t* doc_offsets, int B, int S, int Hq,
                          int Hkv, int D, float rope_theta, llama_attn_bf16* kcache, llama_attn_bf16* vcache,
                          int Lmax, cudaStream_t stream) {
  return prefill_bf16_cached(q, k, v, out, lse, doc_offsets, B, S, Hq, Hkv, D, rope_theta, kcache, vcache, Lmax,
                             QChunks{S, S, 0, 0}, stream);
}

int llama_attn_prefill_cp(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                          llama_attn_bf16* out, float* lse, int B, int Sq, int Skv, int Hq, int Hkv, int D,
                          int q_pos_a, int q_split, int q_pos_b, float rope_theta, cudaStream_t stream) {
  const int st = check_cp(B, Sq, Skv, q_pos_a, q_split, q_pos_b);
  if (st) return st;
  return prefill_bf16_cached(q, k, v, out, lse, nullptr, B, Sq, Hq, Hkv, D, rope_theta, nullptr, nullptr, 0,
                             QChunks{Skv, q_split, q_pos_a, q_pos_b}, stream);
}

int llama_attn_prefill_rotated(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                               llama_attn_bf16* out, float* lse, const int32_t* doc_offsets, int B, int S, int Hq,
                               int Hkv, int D, cudaStream_t stream) {
  return prefill_bf16_cached(q, k, v, out, lse, doc_offsets, B, S, Hq, Hkv, D, 500000.f, nullptr, nullptr, 0,
                             QChunks{S, S, 0, 0}, stream, true);
}

size_t llama_attn_rope_table_size(int maxpos, int D) {
  if (maxpos <= 0 || D < 2 || D > 128 || (D % 2) != 0) return 0;
  return static_cast<size_t>(maxpos) * (D / 2) * sizeof(float2);
}

int llama_attn_rope_table_build(void* table, size_t table_bytes, int maxpos, int D, float rope_theta,
                                cudaStream_t stream) {
  const size_t need = llama_attn_rope_table_size(maxpos, D);
  if (!table || need == 0 || (reinterpret_cast<uintptr_t>(table) & 15u)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (table_bytes < need) return LLAMA_ATTN_ERR_WORKSPACE;
  la::rope_table_kernel<<<grid_for(static_cast<int64_t>(maxpos) * (D / 2), 256), 256, 0, stream>>>(
      static_cast<float2*>(table), maxpos, D, static_cast<double>(rope_theta));
  return cuda_status(cudaGetLastError());
}

size_t llama_attn_prefill_workspace_size(int B, int S, int Hkv, int D) {
  if (B <= 0 || S <= 0 || Hkv <= 0 || D != 128) return 0;
  return prefill_ws_layout(B, S, Hkv).total;
}

int llama_attn_prefill_ws(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                          llama_attn_bf16* out, float* lse, const int32_t* doc_offsets, int B, int S, int Hq,
                          int Hkv, int D, const void* rope_table, int rope_rows, llama_attn_bf16* kcache,
                          llama_attn_bf16* vcache, int Lmax, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream) {
  return prefill_bf16_caller(q, k, v, out, lse, doc_offsets, B, S, Hq, Hkv, D, rope_table, rope_rows, kcache, vcache,
                             Lmax, QChunks{S, S, 0, 0}, workspace, workspace_bytes, stream);
}

int llama_attn_prefill_cp_ws(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                             llama_attn_bf16* out, float* lse, int B, int Sq, int Skv, int Hq, int Hkv, int D,
                             int q_pos_a, int q_split, int q_pos_b, const void* rope_table, int rope_rows,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const int st = check_cp(B, Sq, Skv, q_pos_a, q_split, q_pos_b);
  if (st) return st;
  return prefill_bf16_caller(q, k, v, out, lse, nullptr, B, Sq, Hq, Hkv, D, rope_table, rope_rows, nullptr, nullptr,
                             0, QChunks{Skv, q_split, q_pos_a, q_pos_b}, workspace, workspace_bytes, stream);
}

int llama_attn_quantize_e4m3(const llama_attn_bf16* x, int64_t n, uint8_t* y, float* scale, cudaStream_t stream) {
  if (!x || !y || !scale || n <= 0 || n % 8 != 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(y) & 7u) || (reinterpret_cast<uintptr_t>(scale) & 3u))
    return LLAMA_ATTN_ERR_INVALID_ARG;
  int dev, st;
  if ((st = current_device(&dev))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCache& dc = g_cache[dev];
  if (dc.amax == nullptr) LA_CUDA(cudaMalloc(&dc.amax, 256));
  LA_CUDA(cudaMemsetAsync(dc.amax, 0, sizeof(unsigned int), stream));
  const int64_t nvec = n / 8;
  int n_sm = 148;
  if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0) n_sm = 148;
  const int64_t g = (nvec + 1023) / 1024;  // four vectors per thread step
  const int grid = static_cast<int>(g < 8 * n_sm ? g : 8 * n_sm);
  prof_count(2);
  la::q8::amax_bf16_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(x), nvec, dc.amax);
  LA_CUDA(cudaGetLastError());
  la::q8::quantize_e4m3_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(x), nvec, dc.amax,
                                                           reinterpret_cast<uint2*>(y), scale);
  return cuda_status(cudaGetLastError());
}

int llama_attn_qkv_fp8_rope(const uint8_t* x, const float* s_x, const uint8_t* w, const float* s_w,
                            llama_attn_bf16* q, llama_attn_bf16* k, llama_attn_bf16* v, const int32_t* doc_offsets,
                            int B, int S, int d_model, int Hq, int Hkv, int D, float rope_theta,
                            cudaStream_t stream) {
  if (!x || !s_x || !w || !s_w || !q || !k || !v) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (B <= 0 || S <= 0 || d_model <= 0 || Hq <= 0 || Hkv <= 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (D != 128 || d_model % la::q8::BK != 0) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(w) || !aligned16(q) || !aligned16(k) || !aligned16(v)) return LLAMA_ATTN_ERR_INVALID_ARG;
  const int64_t M = static_cast<int64_t>(B) * S;
  const int64_t n_heads = static_cast<int64_t>(Hq) + 2 * Hkv;
  if (M > INT32_MAX - 1 || n_heads * 128 > INT32_MAX || static_cast<int64_t>(Hq) * 256 >= (int64_t(1) << 32))
    return LLAMA_ATTN_ERR_UNSUPPORTED;
  int dev, st;
  if ((st = current_device(&dev))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCache& dc = g_cache[dev];
  const float2* tab = nullptr;
  if ((st = rope_table(dc, static_cast<double>(rope_theta), D, S, stream, &tab))) return st;
  int n_sm = 148;
  if ((st = device_setup(dev, &n_sm))) return st;
  const int32_t* doc_start = nullptr;
  if (doc_offsets) {
    if ((st = grow(reinterpret_cast<void**>(&dc.doc_start), &dc.doc_bytes, sizeof(int32_t) * M))) return st;
    prof_count(1);
    const int g = grid_for(M, 256);
    la::doc_prep_kernel<<<g < 8 * n_sm ? g : 8 * n_sm, 256, 0, stream>>>(doc_offsets, B, S, dc.doc_start);
    LA_CUDA(cudaGetLastError());
    doc_start = dc.doc_start;
  }
  const int N = static_cast<int>(n_heads * 128);
  CUtensorMap tx, tw, tq, tk, tv;
  if ((st = tmap_2d(&tx, x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, d_model, la::q8::BK, la::q8::BM))) return st;
  if ((st = tmap_2d(&tw, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, d_model, la::q8::BK, la::q8::BN))) return st;
  if ((st = tmap_2d(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, static_cast<int64_t>(Hq) * 128, 64, la::q8::BM)))
    return st;
  if ((st = tmap_2d(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, static_cast<int64_t>(Hkv) * 128, 64, la::q8::BM)))
    return st;
  if ((st = tmap_2d(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, static_cast<int64_t>(Hkv) * 128, 64, la::q8::BM)))
    return st;
  la::q8::Params p;
  p.M = static_cast<int>(M);
  p.K = d_model;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = S;
  p.n_mt = static_cast<int>((M + la::q8::BM - 1) / la::q8::BM);
  p.n_nt = (N + la::q8::BN - 1) / la::q8::BN;
  p.n_kb = d_model / la::q8::BK;
  p.doc_start = doc_start;
  p.rope_tab = reinterpret_cast<const float4*>(tab);
  p.s_x = s_x;
  p.s_w = s_w;
  p.epoch = next_epoch();
  const int64_t tiles = static_cast<int64_t>(p.n_mt) * p.n_nt;
  if (tiles > INT32_MAX) return LLAMA_ATTN_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(tiles < n_sm ? tiles : n_sm);
  prof_count(1);
  const int pair = prof_before(stream);
  la::q8::qkv_fp8_rope_kernel<<<grid, la::q8::NTHREADS, la::q8::SMEM_ALLOC, stream>>>(tx, tw, tq, tk, tv, p);
  const cudaError_t e = cudaGetLastError();
  prof_after(pair, stream);
  return cuda_status(e);
}

int llama_attn_prefill_f32(const float* q, const float* k, const float* v, float* out, const int32_t* doc_offsets,
                           int B, int S, int Hq, int Hkv, int D, float rope_theta, cudaStream_t stream) {
  int st = check_prefill_common(q, k, v, out, B, S, Hq, Hkv, rope_theta);
  if (st) return st;
  if (D < 2 || D > 128 || (D % 2) != 0) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (D != 32 && D != 64 && D != 128 && D != 16 && D != 8) return LLAMA_ATTN_ERR_UNSUPPORTED;
  int dev;
  if ((st = current_device(&dev))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCache& dc = g_cache[dev];
  const float2* tab = nullptr;
  if ((st = rope_table(dc, static_cast<double>(rope_theta), D, S, stream, &tab))) return st;
  const int64_t ntok = static_cast<int64_t>(B) * S;
  int n_sm = 148;
  if ((st = device_setup(dev, &n_sm))) return st;
  const int32_t* doc_start = nullptr;
  if (doc_offsets) {
    if ((st = grow(reinterpret_cast<void**>(&dc.doc_start), &dc.doc_bytes, sizeof(int32_t) * ntok))) return st;
    prof_count(1);
    const int g = grid_for(ntok, 256);
    la::doc_prep_kernel<<<g < 8 * n_sm ? g : 8 * n_sm, 256, 0, stream>>>(doc_offsets, B, S, dc.doc_start);
    LA_CUDA(cudaGetLastError());
    doc_start = dc.doc_start;
  }
  if (B > 65535 || Hq > 65535) return LLAMA_ATTN_ERR_UNSUPPORTED;
  const dim3 grid((S + 63) / 64, Hq, B);
  prof_count(1);
  const int pair = prof_before(stream);
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  switch (D) {
    case 8: la::prefill_f32_kernel<8><<<grid, 64, 0, stream>>>(q, k, v, out, doc_start, tab, S, Hq, Hkv, scale); break;
    case 16: la::prefill_f32_kernel<16><<<grid, 64, 0, stream>>>(q, k, v, out, doc_start, tab, S, Hq, Hkv, scale); break;
    case 32: la::prefill_f32_kernel<32><<<grid, 64, 0, stream>>>(q, k, v, out, doc_start, tab, S, Hq, Hkv, scale); break;
    case 64: la::prefill_f32_kernel<64><<<grid, 64, 0, stream>>>(q, k, v, out, doc_start, tab, S, Hq, Hkv, scale); break;
    default: la::prefill_f32_kernel<128><<<grid, 64, 0, stream>>>(q, k, v, out, doc_start, tab, S, Hq, Hkv, scale); break;
  }
  const cudaError_t e = cudaGetLastError();
  prof_after(pair, stream);
  return cuda_status(e);
}

size_t llama_attn_decode_workspace_size(int B, int Hq, int Lmax, int D) {
  if (B <= 0 || Hq <= 0 || Lmax <= 0 || D != 128) return 0;
  const size_t nchunk = (static_cast<size_t>(Lmax) + la::dec::CHUNK - 1) / la::dec::CHUNK;
  const size_t slots = static_cast<size_t>(B) * Hq * nchunk;
  const size_t o_bytes = slots * 128 * sizeof(float);
  const size_t lse_bytes = slots * sizeof(float);
  return ((o_bytes + lse_bytes + 255) / 256) * 256;
}

}  // extern "C"

namespace {

// Argument checks shared by the decode entry points (before any launch).
int check_decode(const void* q, const void* kc, const void* vc, const int32_t* lens, const void* out, int B, int Hq,
                 int Hkv, int D, float rope_theta) {
  if (!q || !kc || !vc || !lens || !out) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (D != 128 || Hq / Hkv > 16) return LLAMA_ATTN_ERR_UNSUPPORTED;
  // grid (chunks, Hkv, B) and the combine's B * Hq blocks
  if (B > 65535 || Hkv > 65535 || Hq > 65535 || static_cast<int64_t>(B) * Hq > INT32_MAX / 2)
    return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (!aligned16(kc) || !aligned16(vc) || !aligned16(q) || !aligned16(out)) return LLAMA_ATTN_ERR_INVALID_ARG;
  return LLAMA_ATTN_OK;
}

// Split-KV partial attention and the log-sum-exp combine, on `stream`, with
// the partials in `part` (llama_attn_decode_workspace_size bytes). Paged when
// block_table is not null. Launches only: no allocation, no synchronisation.
int decode_launch(const llama_attn_bf16* q, const CUtensorMap& tk, const CUtensorMap& tv, const int32_t* lens,
                  llama_attn_bf16* out, int B, int Hq, int Hkv, int Lmax, float rope_theta, const int32_t* block_table,
                  int page_size, int max_blocks, int n_pages, void* part, cudaStream_t stream) {
  la::dec::Params p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.Lmax = Lmax;
  p.nchunk = (Lmax + la::dec::CHUNK - 1) / la::dec::CHUNK;
  p.lens = lens;
  p.q = q;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  p.epoch = next_epoch();
  p.rope_theta = static_cast<double>(rope_theta);
  p.block_table = block_table;
  p.page_size = page_size;
  p.max_blocks = max_blocks;
  p.n_pages = n_pages;
  const size_t slots = static_cast<size_t>(B) * Hq * p.nchunk;
  p.part_o = static_cast<float*>(part);
  p.part_lse = p.part_o + slots * 128;
  const dim3 grid(p.nchunk, Hkv, B);
  prof_count(2);
  const int pair = prof_before(stream);
  if (block_table)
    la::dec::decode_split_kernel<true><<<grid, la::dec::NTHREADS, la::dec::SMEM_ALLOC, stream>>>(tk, tv, p);
  else
    la::dec::decode_split_kernel<false><<<grid, la::dec::NTHREADS, la::dec::SMEM_ALLOC, stream>>>(tk, tv, p);
  const cudaError_t e = cudaGetLastError();
  prof_after(pair, stream);
  if (e != cudaSuccess) return LLAMA_ATTN_ERR_CUDA;
  la::dec::decode_combine_kernel<<<B * Hq, 128, 0, stream>>>(p.part_o, p.part_lse, lens, out, Hq, Lmax, p.nchunk);
  return cuda_status(cudaGetLastError());
}

}  // namespace

extern "C" {

int llama_attn_decode(const llama_attn_bf16* q, const llama_attn_bf16* kcache, const llama_attn_bf16* vcache,
                      const int32_t* cache_lens, llama_attn_bf16* out, int B, int Hq, int Hkv, int D, int Lmax,
                      float rope_theta, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  int st = check_decode(q, kcache, vcache, cache_lens, out, B, Hq, Hkv, D, rope_theta);
  if (st) return st;
  if (Lmax <= 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * Hkv * Lmax >= INT32_MAX) return LLAMA_ATTN_ERR_UNSUPPORTED;
  const size_t need = llama_attn_decode_workspace_size(B, Hq, Lmax, D);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return LLAMA_ATTN_ERR_WORKSPACE;
  int dev;
  if ((st = current_device(&dev))) return st;
  if ((st = device_setup(dev, nullptr))) return st;
  CUtensorMap tk, tv;
  const int64_t rows = static_cast<int64_t>(B) * Hkv * Lmax;
  if ((st = tmap_rows(&tk, kcache, rows))) return st;
  if ((st = tmap_rows(&tv, vcache, rows))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);  // only the benchmark instrumentation is shared
  return decode_launch(q, tk, tv, cache_lens, out, B, Hq, Hkv, Lmax, rope_theta, nullptr, 0, 0, 0, workspace, stream);
}

int llama_attn_decode_noalloc(const llama_attn_bf16* q, const llama_attn_bf16* kcache,
                              const llama_attn_bf16* vcache, const int32_t* cache_lens, llama_attn_bf16* out, int B,
                              int Hq, int Hkv, int D, int Lmax, float rope_theta, cudaStream_t stream) {
  int st = check_decode(q, kcache, vcache, cache_lens, out, B, Hq, Hkv, D, rope_theta);
  if (st) return st;
  if (Lmax <= 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * Hkv * Lmax >= INT32_MAX) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (llama_attn_decode_workspace_size(B, Hq, Lmax, D) > kNoAllocScratchBytes) return LLAMA_ATTN_ERR_WORKSPACE;
  int dev;
  if ((st = current_device(&dev))) return st;
  if ((st = device_setup(dev, nullptr))) return st;
  CUtensorMap tk, tv;
  const int64_t rows = static_cast<int64_t>(B) * Hkv * Lmax;
  if ((st = tmap_rows(&tk, kcache, rows))) return st;
  if ((st = tmap_rows(&tv, vcache, rows))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_noalloc_scratch_addr[dev] == nullptr) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr) return LLAMA_ATTN_ERR_CUDA;
    g_noalloc_scratch_addr[dev] = addr;
  }
  return decode_launch(q, tk, tv, cache_lens, out, B, Hq, Hkv, Lmax, rope_theta, nullptr, 0, 0, 0,
                       g_noalloc_scratch_addr[dev], stream);
}

int llama_attn_decode_paged(const llama_attn_bf16* q, const llama_attn_bf16* kpages, const llama_attn_bf16* vpages,
                            const int32_t* block_table, const int32_t* cache_lens, llama_attn_bf16* out, int B,
                            int Hq, int Hkv, int D, int page_size, int max_blocks, int n_pages, float rope_theta,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  int st = check_decode(q, kpages, vpages, cache_lens, out, B, Hq, Hkv, D, rope_theta);
  if (st) return st;
  if (!block_table || page_size <= 0 || max_blocks <= 0 || n_pages <= 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (page_size % la::dec::ROWS != 0) return LLAMA_ATTN_ERR_UNSUPPORTED;
  const int64_t Lmax64 = static_cast<int64_t>(max_blocks) * page_size;
  if (Lmax64 >= INT32_MAX || static_cast<int64_t>(n_pages) * Hkv * page_size >= INT32_MAX - page_size)
    return LLAMA_ATTN_ERR_UNSUPPORTED;
  const int Lmax = static_cast<int>(Lmax64);
  const size_t need = llama_attn_decode_workspace_size(B, Hq, Lmax, D);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return LLAMA_ATTN_ERR_WORKSPACE;
  int dev;
  if ((st = current_device(&dev))) return st;
  if ((st = device_setup(dev, nullptr))) return st;
  CUtensorMap tk, tv;
  const int64_t rows = static_cast<int64_t>(n_pages) * Hkv * page_size;
  if ((st = tmap_rows(&tk, kpages, rows))) return st;
  if ((st = tmap_rows(&tv, vpages, rows))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);
  return decode_launch(q, tk, tv, cache_lens, out, B, Hq, Hkv, Lmax, rope_theta, block_table, page_size, max_blocks,
                       n_pages, workspace, stream);
}

}  // extern "C"
