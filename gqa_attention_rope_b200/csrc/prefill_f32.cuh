// prefill_f32.cuh -- grouped-query causal attention with RoPE and the
// cross-document mask in true fp32 arithmetic on CUDA cores.
//
// One thread owns one query row; a block covers 64 rows of one query head.
// Key/value tiles of 64 rows are staged in shared memory, the keys rotated at
// their document positions on the way in. The softmax is taken online over
// chunks of 16 keys with accurate expf (no fast-math), so the result stays
// within ~1e-6 of the float64 definition for unit-variance inputs.
#pragma once

#include "ptx.cuh"

namespace la {

template <int D>
__global__ void __launch_bounds__(64) prefill_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    float* __restrict__ out, const int32_t* __restrict__ doc_start, const float2* __restrict__ tab,
    int S, int Hq, int Hkv, float scale) {
  constexpr int BQ = 64, BK = (D > 64) ? 32 : 64, HALF = D / 2, CH = 16;
  __shared__ float sK[BK][D + 1];
  __shared__ float sV[BK][D + 1];

  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (Hq / Hkv);
  const int tid = threadIdx.x;
  const int64_t rowbase = static_cast<int64_t>(b) * S;
  const int i = qt * BQ + tid;
  const bool valid = i < S;
  const int ic = min(i, S - 1);
  const int ds_i = doc_start ? doc_start[rowbase + ic] : 0;

  // rotated query row
  float qr[D];
  {
    const float* qp = q + ((rowbase + ic) * Hq + h) * D;
    const float2* tp = tab + static_cast<int64_t>(ic - ds_i) * HALF;
#pragma unroll
    for (int kk = 0; kk < HALF; ++kk) {
      const float2 cs = tp[kk];
      const float x0 = qp[2 * kk], x1 = qp[2 * kk + 1];
      qr[2 * kk] = x0 * cs.x - x1 * cs.y;
      qr[2 * kk + 1] = x0 * cs.y + x1 * cs.x;
    }
  }

  const int q0 = qt * BQ;
  const int ds_first = doc_start ? doc_start[rowbase + q0] : 0;
  const int kt_lo = ds_first / BK, kt_hi = min(q0 + BQ - 1, S - 1) / BK;  // key tiles to visit

  float m = -INFINITY, l = 0.f;
  float o[D];
#pragma unroll
  for (int d = 0; d < D; ++d) o[d] = 0.f;

  for (int kt = kt_lo; kt <= kt_hi; ++kt) {
    const int kb = kt * BK;
    for (int jj = tid; jj < BK; jj += BQ) {
      const int j = kb + jj;
      if (j < S) {
        const int64_t tok = rowbase + j;
        const int pos_j = j - (doc_start ? doc_start[tok] : 0);
        const float* kp = k + (tok * Hkv + g) * D;
        const float* vp = v + (tok * Hkv + g) * D;
        const float2* tp = tab + static_cast<int64_t>(pos_j) * HALF;
        for (int kk = 0; kk < HALF; ++kk) {
          const float2 cs = tp[kk];
          const float x0 = kp[2 * kk], x1 = kp[2 * kk + 1];
          sK[jj][2 * kk] = x0 * cs.x - x1 * cs.y;
          sK[jj][2 * kk + 1] = x0 * cs.y + x1 * cs.x;
        }
        for (int d = 0; d < D; ++d) sV[jj][d] = vp[d];
      } else {
        for (int d = 0; d < D; ++d) sK[jj][d] = 0.f, sV[jj][d] = 0.f;
      }
    }
    __syncthreads();
    const int lo = ds_i - kb, hi = ic - kb;  // visible key columns: lo <= c <= hi
    for (int c0 = 0; c0 < BK; c0 += CH) {
      if (c0 > hi || c0 + CH - 1 < lo) continue;
      float s[CH];
      float cmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int cc = c0 + c;
        if (cc < lo || cc > hi) {
          s[c] = -INFINITY;
          continue;
        }
        float dot = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) dot = fmaf(qr[d], sK[cc][d], dot);
        s[c] = dot * scale;
        cmax = fmaxf(cmax, s[c]);
      }
      const float m_new = fmaxf(m, cmax);
      const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
      l *= alpha;
#pragma unroll
      for (int d = 0; d < D; ++d) o[d] *= alpha;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        if (s[c] == -INFINITY) continue;
        const float pc = expf(s[c] - m_new);
        l += pc;
        const int cc = c0 + c;
#pragma unroll
        for (int d = 0; d < D; ++d) o[d] = fmaf(pc, sV[cc][d], o[d]);
      }
      m = m_new;
    }
    __syncthreads();
  }
  if (valid) {
    float* op = out + ((rowbase + i) * Hq + h) * D;
    const float inv = 1.f / l;
#pragma unroll
    for (int d = 0; d < D; ++d) op[d] = o[d] * inv;
  }
}

}  // namespace la
