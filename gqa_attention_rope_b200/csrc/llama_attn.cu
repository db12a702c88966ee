// llama_attn.cu -- the library's single translation unit: host-side argument
// checks, TMA descriptor encoding, per-device caches (RoPE tables, scratch) and
// kernel launches behind the C ABI declared in include/llama_attn.h.
#include <cudaTypedefs.h>

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

#define LLAMA_ATTN_VERSION 200  // 0.2.0: context-parallel, pre-rotated and FP8 projection entry points

namespace {

constexpr int kMaxDevices = 64;

struct RopeTable {
  double theta = 0.0;
  int D = 0;
  int maxpos = 0;
  float2* ptr = nullptr;
};

struct DeviceCache {
  std::vector<RopeTable> tables;
  void* krot = nullptr;
  size_t krot_bytes = 0;
  int32_t* doc_start = nullptr;
  size_t doc_bytes = 0;
  int* sched = nullptr;  // work-item counter of the persistent prefill kernel
  bool prefill_attr_set = false;
  bool decode_attr_set = false;
  bool decode_paged_attr_set = false;
  unsigned int* amax = nullptr;  // per-tensor amax of the E4M3 quantizer
  bool qkv_attr_set = false;
};

std::mutex g_mutex;
DeviceCache g_cache[kMaxDevices];
unsigned int g_epoch = 0;

// Distinct, nonzero id per launch that uses bounded waits.
unsigned int next_epoch() {
  if (++g_epoch == 0) ++g_epoch;
  return g_epoch;
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
bool g_noalloc_attr_set[kMaxDevices];
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
    case LLAMA_ATTN_ERR_WORKSPACE: return "decode workspace missing, misaligned or too small";
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

// bf16 prefill shared by llama_attn_prefill and llama_attn_prefill_ex: lse,
// kcache and vcache may be null (no log-sum-exp output, no cache append).
// Query chunks (context parallelism): q holds S rows per batch row, rows
// [0, q_split) at global positions q_pos_a.., rows [q_split, S) at q_pos_b..;
// k and v hold the whole sequence, Skv rows. A plain prefill is
// Skv = q_split = S, q_pos_a = q_pos_b = 0.
struct QChunks {
  int Skv, q_split, q_pos_a, q_pos_b;
};

int prefill_bf16_impl(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                      llama_attn_bf16* out, float* lse, const int32_t* doc_offsets, int B, int S, int Hq, int Hkv,
                      int D, float rope_theta, llama_attn_bf16* kcache, llama_attn_bf16* vcache, int Lmax,
                      const QChunks& qc, cudaStream_t stream, bool prerotated = false) {
  int st = check_prefill_common(q, k, v, out, B, S, Hq, Hkv, rope_theta);
  if (st) return st;
  const int Skv = qc.Skv;
  if (Skv <= 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * Skv > INT32_MAX) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (D != 128) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if ((kcache == nullptr) != (vcache == nullptr)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (kcache && (Lmax < S || !aligned16(kcache) || !aligned16(vcache))) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(S) * Hq * 256 >= (int64_t(1) << 40)) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(Skv) * Hkv * 256 >= (int64_t(1) << 40)) return LLAMA_ATTN_ERR_UNSUPPORTED;
  int dev;
  if ((st = current_device(&dev))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCache& dc = g_cache[dev];

  const float2* tab = nullptr;
  const int n_pos = S > Skv ? S : Skv;
  if (!prerotated && (st = rope_table(dc, static_cast<double>(rope_theta), D, n_pos, stream, &tab))) return st;
  const int64_t ntok = static_cast<int64_t>(B) * S;
  const int64_t nkv_tok = static_cast<int64_t>(B) * Skv;
  const int32_t* doc_start = nullptr;
  if (doc_offsets) {
    if ((st = grow(reinterpret_cast<void**>(&dc.doc_start), &dc.doc_bytes, sizeof(int32_t) * ntok))) return st;
    prof_count(1);
    la::doc_prep_kernel<<<1, 1024, 0, stream>>>(doc_offsets, B, S, dc.doc_start);
    LA_CUDA(cudaGetLastError());
    doc_start = dc.doc_start;
  }
  const size_t kbytes = static_cast<size_t>(nkv_tok) * Hkv * 128 * 2;
  if (!prerotated && (st = grow(&dc.krot, &dc.krot_bytes, kbytes))) return st;
  const int64_t nvec = ntok * Hkv * 16;
  const int64_t nvec_kv = nkv_tok * Hkv * 16;
  const void* k_rot = k;  // pre-rotated keys are read as given
  if (!prerotated) {
    prof_count(1);
    la::rope_rotate_rows_bf16_kernel<<<grid_for(nvec_kv, 256), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(k), reinterpret_cast<uint4*>(dc.krot), reinterpret_cast<const float4*>(tab),
        doc_start, Skv, Hkv, nvec_kv);
    LA_CUDA(cudaGetLastError());
    k_rot = dc.krot;
  }
  if (kcache) {
    prof_count(1);
    la::kv_cache_append_kernel<<<grid_for(nvec, 256), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v), reinterpret_cast<const float4*>(tab),
        doc_start, reinterpret_cast<uint4*>(kcache), reinterpret_cast<uint4*>(vcache), S, Hkv, Lmax, nvec);
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
  p.doc_start = doc_start;
  p.rope_tab = reinterpret_cast<const float4*>(tab);
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  p.epoch = next_epoch();
  if (dc.sched == nullptr) LA_CUDA(cudaMalloc(&dc.sched, 256));
  LA_CUDA(cudaMemsetAsync(dc.sched, 0, sizeof(int), stream));
  p.sched = dc.sched;
  p.lse = lse;
  const int64_t items = static_cast<int64_t>(B) * p.n_qt * p.n_hp;
  if (items > INT32_MAX) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (!dc.prefill_attr_set) {
    LA_CUDA(cudaFuncSetAttribute(la::pfx::prefill_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 la::pfx::SMEM_ALLOC));
    dc.prefill_attr_set = true;
  }
  prof_count(1);
  const int pair = prof_before(stream);
  int n_sm = 148;
  if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0) n_sm = 148;
  const int grid = static_cast<int>(items < n_sm ? items : n_sm);
  la::pfx::prefill_bf16_kernel<<<grid, la::pfx::NTHREADS, la::pfx::SMEM_ALLOC, stream>>>(tq, tk, tv, to, p);
  const cudaError_t e = cudaGetLastError();
  prof_after(pair, stream);
  return cuda_status(e);
}

}  // namespace

extern "C" {

int llama_attn_prefill(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                       llama_attn_bf16* out, const int32_t* doc_offsets, int B, int S, int Hq, int Hkv, int D,
                       float rope_theta, cudaStream_t stream) {
  return prefill_bf16_impl(q, k, v, out, nullptr, doc_offsets, B, S, Hq, Hkv, D, rope_theta, nullptr, nullptr, 0,
                           QChunks{S, S, 0, 0}, stream);
}

int llama_attn_prefill_ex(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                          llama_attn_bf16* out, float* lse, const int32_t* doc_offsets, int B, int S, int Hq,
                          int Hkv, int D, float rope_theta, llama_attn_bf16* kcache, llama_attn_bf16* vcache,
                          int Lmax, cudaStream_t stream) {
  return prefill_bf16_impl(q, k, v, out, lse, doc_offsets, B, S, Hq, Hkv, D, rope_theta, kcache, vcache, Lmax,
                           QChunks{S, S, 0, 0}, stream);
}

int llama_attn_prefill_cp(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                          llama_attn_bf16* out, float* lse, int B, int Sq, int Skv, int Hq, int Hkv, int D,
                          int q_pos_a, int q_split, int q_pos_b, float rope_theta, cudaStream_t stream) {
  if (B <= 0 || Sq <= 0 || Skv <= 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  constexpr int kT = la::pfx::BM;
  if (q_split < 0 || q_split > Sq || q_pos_a < 0 || q_pos_b < 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (q_split % kT != 0 || q_pos_a % kT != 0 || q_pos_b % kT != 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(q_pos_a) + q_split > Skv) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(q_pos_b) + (Sq - q_split) > Skv) return LLAMA_ATTN_ERR_INVALID_ARG;
  return prefill_bf16_impl(q, k, v, out, lse, nullptr, B, Sq, Hq, Hkv, D, rope_theta, nullptr, nullptr, 0,
                           QChunks{Skv, q_split, q_pos_a, q_pos_b}, stream);
}

int llama_attn_prefill_rotated(const llama_attn_bf16* q, const llama_attn_bf16* k, const llama_attn_bf16* v,
                               llama_attn_bf16* out, float* lse, const int32_t* doc_offsets, int B, int S, int Hq,
                               int Hkv, int D, cudaStream_t stream) {
  return prefill_bf16_impl(q, k, v, out, lse, doc_offsets, B, S, Hq, Hkv, D, 500000.f, nullptr, nullptr, 0,
                           QChunks{S, S, 0, 0}, stream, true);
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
  const int32_t* doc_start = nullptr;
  if (doc_offsets) {
    if ((st = grow(reinterpret_cast<void**>(&dc.doc_start), &dc.doc_bytes, sizeof(int32_t) * M))) return st;
    prof_count(1);
    la::doc_prep_kernel<<<1, 1024, 0, stream>>>(doc_offsets, B, S, dc.doc_start);
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
  if (!dc.qkv_attr_set) {
    LA_CUDA(cudaFuncSetAttribute(la::q8::qkv_fp8_rope_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 la::q8::SMEM_ALLOC));
    dc.qkv_attr_set = true;
  }
  int n_sm = 148;
  if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0) n_sm = 148;
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
  const int32_t* doc_start = nullptr;
  if (doc_offsets) {
    if ((st = grow(reinterpret_cast<void**>(&dc.doc_start), &dc.doc_bytes, sizeof(int32_t) * ntok))) return st;
    prof_count(1);
    la::doc_prep_kernel<<<1, 1024, 0, stream>>>(doc_offsets, B, S, dc.doc_start);
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

int llama_attn_decode(const llama_attn_bf16* q, const llama_attn_bf16* kcache, const llama_attn_bf16* vcache,
                      const int32_t* cache_lens, llama_attn_bf16* out, int B, int Hq, int Hkv, int D, int Lmax,
                      float rope_theta, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !kcache || !vcache || !cache_lens || !out) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || Hq % Hkv != 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (D != 128 || Hq / Hkv > 16) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535 || B * Hq > INT32_MAX / 2) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * Hkv * Lmax >= INT32_MAX) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (!aligned16(kcache) || !aligned16(vcache) || !aligned16(q) || !aligned16(out)) return LLAMA_ATTN_ERR_INVALID_ARG;
  const size_t need = llama_attn_decode_workspace_size(B, Hq, Lmax, D);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return LLAMA_ATTN_ERR_WORKSPACE;
  int dev, st;
  if ((st = current_device(&dev))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCache& dc = g_cache[dev];
  const float2* tab = nullptr;
  if ((st = rope_table(dc, static_cast<double>(rope_theta), D, Lmax + 1, stream, &tab))) return st;

  CUtensorMap tk, tv;
  const int64_t rows = static_cast<int64_t>(B) * Hkv * Lmax;
  if ((st = tmap_rows(&tk, kcache, rows))) return st;
  if ((st = tmap_rows(&tv, vcache, rows))) return st;

  la::dec::Params p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.Lmax = Lmax;
  p.nchunk = (Lmax + la::dec::CHUNK - 1) / la::dec::CHUNK;
  p.lens = cache_lens;
  p.q = q;
  p.rope_tab = reinterpret_cast<const float4*>(tab);
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  p.epoch = next_epoch();
  p.rope_theta = static_cast<double>(rope_theta);
  const size_t slots = static_cast<size_t>(B) * Hq * p.nchunk;
  p.part_o = static_cast<float*>(workspace);
  p.part_lse = p.part_o + slots * 128;
  if (!dc.decode_attr_set) {
    LA_CUDA(cudaFuncSetAttribute(la::dec::decode_split_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 la::dec::SMEM_ALLOC));
    dc.decode_attr_set = true;
  }
  const dim3 grid(p.nchunk, Hkv, B);
  prof_count(2);
  const int pair = prof_before(stream);
  la::dec::decode_split_kernel<false><<<grid, la::dec::NTHREADS, la::dec::SMEM_ALLOC, stream>>>(tk, tv, p);
  const cudaError_t e = cudaGetLastError();
  prof_after(pair, stream);
  if (e != cudaSuccess) return LLAMA_ATTN_ERR_CUDA;
  la::dec::decode_combine_kernel<<<B * Hq, 128, 0, stream>>>(p.part_o, p.part_lse, cache_lens, out, Hq, Lmax,
                                                            p.nchunk);
  return cuda_status(cudaGetLastError());
}

int llama_attn_decode_noalloc(const llama_attn_bf16* q, const llama_attn_bf16* kcache,
                              const llama_attn_bf16* vcache, const int32_t* cache_lens, llama_attn_bf16* out, int B,
                              int Hq, int Hkv, int D, int Lmax, float rope_theta, cudaStream_t stream) {
  if (!q || !kcache || !vcache || !cache_lens || !out) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || Hq % Hkv != 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (D != 128 || Hq / Hkv > 16) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535 || B * Hq > INT32_MAX / 2) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * Hkv * Lmax >= INT32_MAX) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (!aligned16(kcache) || !aligned16(vcache) || !aligned16(q) || !aligned16(out)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (llama_attn_decode_workspace_size(B, Hq, Lmax, D) > kNoAllocScratchBytes) return LLAMA_ATTN_ERR_WORKSPACE;
  int dev, st;
  if ((st = current_device(&dev))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_noalloc_scratch_addr[dev] == nullptr) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr) return LLAMA_ATTN_ERR_CUDA;
    g_noalloc_scratch_addr[dev] = addr;
  }
  if (!g_noalloc_attr_set[dev]) {
    LA_CUDA(cudaFuncSetAttribute(la::dec::decode_split_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 la::dec::SMEM_ALLOC_SELF_TABLE));
    g_noalloc_attr_set[dev] = true;
  }
  CUtensorMap tk, tv;
  const int64_t rows = static_cast<int64_t>(B) * Hkv * Lmax;
  if ((st = tmap_rows(&tk, kcache, rows))) return st;
  if ((st = tmap_rows(&tv, vcache, rows))) return st;

  la::dec::Params p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.Lmax = Lmax;
  p.nchunk = (Lmax + la::dec::CHUNK - 1) / la::dec::CHUNK;
  p.lens = cache_lens;
  p.q = q;
  p.rope_tab = nullptr;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  p.epoch = next_epoch();
  p.rope_theta = static_cast<double>(rope_theta);
  const size_t slots = static_cast<size_t>(B) * Hq * p.nchunk;
  p.part_o = static_cast<float*>(g_noalloc_scratch_addr[dev]);
  p.part_lse = p.part_o + slots * 128;
  const dim3 grid(p.nchunk, Hkv, B);
  la::dec::decode_split_kernel<true><<<grid, la::dec::NTHREADS, la::dec::SMEM_ALLOC_SELF_TABLE, stream>>>(tk, tv, p);
  LA_CUDA(cudaGetLastError());
  la::dec::decode_combine_kernel<<<B * Hq, 128, 0, stream>>>(p.part_o, p.part_lse, cache_lens, out, Hq, Lmax,
                                                            p.nchunk);
  return cuda_status(cudaGetLastError());
}

int llama_attn_decode_paged(const llama_attn_bf16* q, const llama_attn_bf16* kpages, const llama_attn_bf16* vpages,
                            const int32_t* block_table, const int32_t* cache_lens, llama_attn_bf16* out, int B,
                            int Hq, int Hkv, int D, int page_size, int max_blocks, int n_pages, float rope_theta,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !kpages || !vpages || !block_table || !cache_lens || !out) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (page_size <= 0 || max_blocks <= 0 || n_pages <= 0) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta)) return LLAMA_ATTN_ERR_INVALID_ARG;
  if (D != 128 || Hq / Hkv > 16 || page_size % la::dec::ROWS != 0) return LLAMA_ATTN_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535 || B * Hq > INT32_MAX / 2) return LLAMA_ATTN_ERR_UNSUPPORTED;
  const int64_t Lmax64 = static_cast<int64_t>(max_blocks) * page_size;
  if (Lmax64 >= INT32_MAX || static_cast<int64_t>(n_pages) * Hkv * page_size >= INT32_MAX - page_size)
    return LLAMA_ATTN_ERR_UNSUPPORTED;
  const int Lmax = static_cast<int>(Lmax64);
  if (!aligned16(kpages) || !aligned16(vpages) || !aligned16(q) || !aligned16(out)) return LLAMA_ATTN_ERR_INVALID_ARG;
  const size_t need = llama_attn_decode_workspace_size(B, Hq, Lmax, D);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return LLAMA_ATTN_ERR_WORKSPACE;
  int dev, st;
  if ((st = current_device(&dev))) return st;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCache& dc = g_cache[dev];
  const float2* tab = nullptr;
  if ((st = rope_table(dc, static_cast<double>(rope_theta), D, Lmax + 1, stream, &tab))) return st;

  CUtensorMap tk, tv;
  const int64_t rows = static_cast<int64_t>(n_pages) * Hkv * page_size;
  if ((st = tmap_rows(&tk, kpages, rows))) return st;
  if ((st = tmap_rows(&tv, vpages, rows))) return st;

  la::dec::Params p;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.Lmax = Lmax;
  p.nchunk = (Lmax + la::dec::CHUNK - 1) / la::dec::CHUNK;
  p.lens = cache_lens;
  p.q = q;
  p.rope_tab = reinterpret_cast<const float4*>(tab);
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  p.epoch = next_epoch();
  p.rope_theta = static_cast<double>(rope_theta);
  p.block_table = block_table;
  p.page_size = page_size;
  p.max_blocks = max_blocks;
  p.n_pages = n_pages;
  const size_t slots = static_cast<size_t>(B) * Hq * p.nchunk;
  p.part_o = static_cast<float*>(workspace);
  p.part_lse = p.part_o + slots * 128;
  if (!dc.decode_paged_attr_set) {
    LA_CUDA(cudaFuncSetAttribute(la::dec::decode_split_kernel<false, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, la::dec::SMEM_ALLOC));
    dc.decode_paged_attr_set = true;
  }
  const dim3 grid(p.nchunk, Hkv, B);
  prof_count(2);
  const int pair = prof_before(stream);
  la::dec::decode_split_kernel<false, true><<<grid, la::dec::NTHREADS, la::dec::SMEM_ALLOC, stream>>>(tk, tv, p);
  const cudaError_t e = cudaGetLastError();
  prof_after(pair, stream);
  if (e != cudaSuccess) return LLAMA_ATTN_ERR_CUDA;
  la::dec::decode_combine_kernel<<<B * Hq, 128, 0, stream>>>(p.part_o, p.part_lse, cache_lens, out, Hq, Lmax,
                                                            p.nchunk);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"
