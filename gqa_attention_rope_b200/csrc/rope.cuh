// rope.cuh -- RoPE cos/sin table, per-token document layout, and the K
// rotation pass that feeds the tensor-core prefill.
//
// RoPE ("Llama 3.1 Architecture: Dense Scaling to 405B and 128K Context",
// "Context Expansion", "High Base Frequency"): theta_k = base^(-2k/D),
// k in [0, D/2 - 1]; the pair (x_2k, x_2k+1) of a token at position p turns by
// p * theta_k (RoFormer rotation). Cross-document mask ("The Llama 3 Herd of
// Models", architecture chapter): positions restart at each document.
#pragma once

#include "ptx.cuh"

namespace la {

// tab[p * (D/2) + k] = (cos(p * theta_k), sin(p * theta_k)) for p < maxpos.
// The angle is formed and reduced in float64 and only the result is rounded
// to float32: a float32 product p * theta_k would be off by ~4e-3 rad at
// p ~ 1.3e5.
__global__ void rope_table_kernel(float2* __restrict__ tab, int maxpos, int D, double base) {
  const int half = D / 2;
  const int64_t n = static_cast<int64_t>(maxpos) * half;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i / half), k = static_cast<int>(i % half);
    const double freq = pow(base, -2.0 * static_cast<double>(k) / static_cast<double>(D));
    double s, c;
    sincos(static_cast<double>(p) * freq, &s, &c);
    tab[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

// Document layout from doc_offsets (cumulative starts in flattened B*S
// coordinates, ending with the sentinel B*S; the count is implicit, so an
// entry may only be read once every earlier one is known to be below B*S).
//
// doc_count: the number of documents n (offs[n] == B*S), or -1 when the array
// is malformed (not starting at 0, not strictly increasing, a document
// crossing a batch-row boundary, an entry past B*S). One thread walks the
// entries in order; they are few (one per document) and after the first miss
// they come from L1.
__device__ __forceinline__ int doc_count(const int32_t* __restrict__ offs, int B, int S) {
  const int64_t total = static_cast<int64_t>(B) * S;
  if (offs[0] != 0) return -1;
  int64_t prev = 0;
  for (int64_t d = 1; d <= total; ++d) {
    const int64_t o = offs[d];
    if (o <= prev || o > total || (prev / S) != ((o - 1) / S)) return -1;
    if (o == total) return static_cast<int>(d);
    prev = o;
  }
  return -1;
}

// Row-local start of the document holding token t (0 when n <= 0: a malformed
// array makes every row one document, so later indexing stays in bounds).
__device__ __forceinline__ int32_t doc_start_of(const int32_t* __restrict__ offs, int n, int64_t t, int S) {
  if (n <= 0) return 0;
  int lo = 0, hi = n - 1;  // largest d with offs[d] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offs[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return static_cast<int32_t>(offs[lo] - (t / S) * S);
}

// Block-wide document count: thread 0 walks, everyone gets the result; a
// malformed array raises LLAMA_ATTN_DEVERR_DOC_OFFSETS (from every block that
// sees it; the bit is the same).
__device__ __forceinline__ int block_doc_count(const int32_t* __restrict__ offs, int B, int S) {
  __shared__ int s_ndocs;
  if (threadIdx.x == 0) {
    const int n = doc_count(offs, B, S);
    if (n < 0) raise_error(LLAMA_ATTN_DEVERR_DOC_OFFSETS);
    s_ndocs = n;
  }
  __syncthreads();
  return s_ndocs;
}

// Per-token row-local document start, doc_start[t] for t < B*S. Grid-stride
// over tokens, any number of blocks.
__global__ void doc_prep_kernel(const int32_t* __restrict__ offs, int B, int S, int32_t* __restrict__ doc_start) {
  const int n = block_doc_count(offs, B, S);
  const int64_t total = static_cast<int64_t>(B) * S;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x)
    doc_start[t] = doc_start_of(offs, n, t, S);
}

// Rotate one bf16 pair (low half = element 2k, high half = element 2k+1).
__device__ __forceinline__ uint32_t rope_rotate_pair(uint32_t xv, float c, float s) {
  const float2 x = unpack_bf16x2(xv);
  return pack_bf16x2(x.x * c - x.y * s, x.x * s + x.y * c);
}

// y = RoPE(x) for x [B, S, H, 128] bf16 at each token's document position.
// One thread per 16-byte vector (4 pairs); the table row of the token is read
// as float4s (2 pairs each). Document positions come either from doc_start
// (when offs is null) or, when offs is given, from the offsets themselves;
// the pass then also writes doc_start_out[t] (if not null) for every token,
// so the attention kernel needs no separate layout pass. offs == null and
// doc_start == null: each batch row is one document.
__global__ void rope_rotate_rows_bf16_kernel(const uint4* __restrict__ x, uint4* __restrict__ y,
                                             const float4* __restrict__ tab,
                                             const int32_t* __restrict__ doc_start,
                                             const int32_t* __restrict__ offs,
                                             int32_t* __restrict__ doc_start_out, int B, int S, int H,
                                             int64_t n_vec) {
  constexpr int kVecPerRow = 16;  // 128 bf16 per head row
  const int n = offs ? block_doc_count(offs, B, S) : 0;
  const int64_t per_tok = static_cast<int64_t>(H) * kVecPerRow;
  for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < n_vec;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = v / per_tok;
    const int c = static_cast<int>(v % kVecPerRow);
    const int i = static_cast<int>(t % S);
    int32_t ds = 0;
    if (offs) {
      ds = doc_start_of(offs, n, t, S);
      if (doc_start_out && v % per_tok == 0) doc_start_out[t] = ds;
    } else if (doc_start) {
      ds = doc_start[t];
    }
    const int pos = i - ds;
    const float4* tp = tab + static_cast<int64_t>(pos) * 32 + c * 2;
    const float4 cs0 = __ldg(tp), cs1 = __ldg(tp + 1);
    uint4 xv = x[v];
    xv.x = rope_rotate_pair(xv.x, cs0.x, cs0.y);
    xv.y = rope_rotate_pair(xv.y, cs0.z, cs0.w);
    xv.z = rope_rotate_pair(xv.z, cs1.x, cs1.y);
    xv.w = rope_rotate_pair(xv.w, cs1.z, cs1.w);
    y[v] = xv;
  }
}

// Appends a prefill batch to a decode-layout KV cache: token i of batch row b
// and KV head h goes to cache row i of (b, h), the key rotated at the token's
// document position (position i when the row is one document), the value
// copied. k, v: [B, S, H, 128]; kcache, vcache: [B, H, Lmax, 128], Lmax >= S.
// One thread per 16-byte vector (4 pairs).
__global__ void kv_cache_append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                       const float4* __restrict__ tab, const int32_t* __restrict__ doc_start,
                                       uint4* __restrict__ kcache, uint4* __restrict__ vcache, int S, int H,
                                       int Lmax, int64_t n_vec) {
  constexpr int kVecPerRow = 16;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n_vec;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = idx / (static_cast<int64_t>(H) * kVecPerRow);
    const int rem = static_cast<int>(idx % (static_cast<int64_t>(H) * kVecPerRow));
    const int h = rem / kVecPerRow, c = rem % kVecPerRow;
    const int64_t b = t / S;
    const int i = static_cast<int>(t % S);
    const int pos = i - (doc_start ? doc_start[t] : 0);
    const float4* tp = tab + static_cast<int64_t>(pos) * 32 + c * 2;
    const float4 cs0 = __ldg(tp), cs1 = __ldg(tp + 1);
    uint4 kv = k[idx];
    kv.x = rope_rotate_pair(kv.x, cs0.x, cs0.y);
    kv.y = rope_rotate_pair(kv.y, cs0.z, cs0.w);
    kv.z = rope_rotate_pair(kv.z, cs1.x, cs1.y);
    kv.w = rope_rotate_pair(kv.w, cs1.z, cs1.w);
    const int64_t dst = ((b * H + h) * Lmax + i) * kVecPerRow + c;
    kcache[dst] = kv;
    vcache[dst] = v[idx];
  }
}

}  // namespace la
