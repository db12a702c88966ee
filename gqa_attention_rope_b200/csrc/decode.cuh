// decode.cuh -- single-token GQA decode against a KV cache, split along the
// cache length, with a log-sum-exp combine.
//
// The query heads of one KV group (G <= 16) are packed as the 16 rows of an
// m16n8k16 bf16 MMA tile, so each cached K/V row is read from HBM once and
// used by every head of its group (the KV-cache saving that motivates GQA on
// "How Meta's Llama 3.1 405B Architecture Actually Works", GQA paragraph).
// Decode does 8 FLOP per cached byte, so the bound is HBM bandwidth; the warp
// MMA is only there to keep the arithmetic off the FP32 pipe.
//
// decode_split_kernel: grid (chunk, kv head, sequence); a CTA covers up to
// CHUNK cache rows. Warp 4 streams 64-row K/V stages with TMA (2D tensor map
// over the [B*Hkv*Lmax, 128] cache, 128B swizzle) through a 3-stage ring; warps
// 0-3 each take 16 rows of every stage: S = q K^T (ldmatrix + mma), mask past
// len, online softmax with quad shuffles, O += P V (P reused from the score
// fragments, V via ldmatrix.trans). The four warps' partials are merged in
// shared memory and the chunk's normalised O and log2-sum-exp are written to
// the workspace.
// decode_combine_kernel: one block per (sequence, query head) merges the
// chunks: out = sum_c 2^(lse_c - M) O_c / sum_c 2^(lse_c - M).
#pragma once

#include "ptx.cuh"
#include "rope.cuh"

namespace la {
namespace dec {

constexpr int CHUNK = 1024;
constexpr int ROWS = 64;
constexpr int NSTAGE = 3;
constexpr int NCW = 4;
constexpr int NTHREADS = (NCW + 1) * 32;
constexpr uint32_t KHALF = ROWS * 128;      // 64 rows x 64 bf16 = 8 KB
constexpr uint32_t STAGE = 4 * KHALF;       // K (2 halves) + V (2 halves)
constexpr uint32_t OFF_BAR = NSTAGE * STAGE;
// The CTA's (cos, sin) row at position len sits after the barriers.
constexpr uint32_t OFF_ROPE_ROW = OFF_BAR + 64;
constexpr uint32_t SMEM_ALLOC = OFF_ROPE_ROW + 64 * 8 + 1024;
static_assert(NCW * (2 * 16 + 16 * 128) * 4 <= OFF_BAR, "combine scratch fits in the ring");

struct Params {
  int B, Hq, Hkv, G, Lmax, nchunk;
  const int32_t* lens;
  const uint16_t* q;         // [B, Hq, 128] bf16 bits
  float scale_log2;
  float* part_o;             // [B, Hq, nchunk, 128]
  float* part_lse;           // [B, Hq, nchunk]
  unsigned int epoch;        // launch id for bounded-wait abort propagation
  double rope_theta;         // RoPE base; the CTA forms the (cos, sin) row of position len itself
  // paged cache (kPaged): logical row n of sequence b lives in page
  // block_table[b * max_blocks + n / page_size] at row n % page_size; the page
  // pool is [n_pages, Hkv, page_size, 128], page_size a multiple of ROWS.
  const int32_t* block_table;
  int page_size, max_blocks, n_pages;
};

__device__ __forceinline__ int valid_len(int len, int Lmax) { return (len < 0 || len > Lmax) ? 0 : len; }

// The query is rotated at position len: the CTA forms that one (cos, sin) row
// itself (float64 angle, the formula of rope_table_kernel) in shared memory,
// so the decode needs no table. The compute warps build it after the block
// barrier, so the producer's first loads are not held back by it.
template <bool kPaged = false>
__global__ void __launch_bounds__(NTHREADS, 2)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + OFF_BAR;
  auto full = [&](uint32_t s) { return bar0 + 8u * s; };
  auto empty = [&](uint32_t s) { return bar0 + 8u * (NSTAGE + s); };

  const int c = blockIdx.x, gk = blockIdx.y, b = blockIdx.z;
  const int len = valid_len(p.lens[b], p.Lmax);
  const int n0 = c * CHUNK;
  if (n0 >= len) return;
  const int n1 = min(len, n0 + CHUNK);
  const int nst = (n1 - n0 + ROWS - 1) / ROWS;
  const int row0 = kPaged ? 0 : (b * p.Hkv + gk) * p.Lmax + n0;  // contiguous layout only
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtx wc{p.epoch};

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), NCW);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  __syncthreads();

  if (warp == NCW) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nst; ++i) {
        const uint32_t st = i % NSTAGE, use = i / NSTAGE;
        if (use > 0 && !mbar_wait(empty(st), (use - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(full(st), STAGE);
        const uint32_t dst = sbase + st * STAGE;
        int r = row0 + i * ROWS;
        if constexpr (kPaged) {
          // a stage of ROWS rows lies inside one page (page_size is a multiple of ROWS)
          const int n = n0 + i * ROWS;
          const int page = p.block_table[static_cast<int64_t>(b) * p.max_blocks + n / p.page_size];
          if (page < 0 || page >= p.n_pages) {
            raise_error(LLAMA_ATTN_DEVERR_BLOCK_TABLE);
            r = p.n_pages * p.Hkv * p.page_size;  // past the pool: TMA reads zeros
          } else {
            r = (page * p.Hkv + gk) * p.page_size + n % p.page_size;
          }
        }
        tma_load_2d(dst, &tm_k, full(st), 0, r);
        tma_load_2d(dst + KHALF, &tm_k, full(st), 64, r);
        tma_load_2d(dst + 2 * KHALF, &tm_v, full(st), 0, r);
        tma_load_2d(dst + 3 * KHALF, &tm_v, full(st), 64, r);
        ++issued;
      }
      for (int st = 0; st < NSTAGE; ++st)
        if (issued > st) mbar_wait(full(st), ((issued - 1 - st) / NSTAGE) & 1, wc);
    }
    return;
  }

  // ---------------------------------------------------------------- compute warps
  const int gq = lane >> 2, t = lane & 3;  // fragment row group / thread-in-group
  const int G = p.G;
  // A fragments of the rotated query: rows = heads of the group (row >= G is zero).
  if (threadIdx.x < 64) {
    const double freq = pow(p.rope_theta, -2.0 * static_cast<double>(threadIdx.x) / 128.0);
    double sn, cs;
    sincos(static_cast<double>(len) * freq, &sn, &cs);
    reinterpret_cast<float2*>(smem + OFF_ROPE_ROW)[threadIdx.x] =
        make_float2(static_cast<float>(cs), static_cast<float>(sn));
  }
  asm volatile("bar.sync 2, %0;" ::"r"(NCW * 32) : "memory");  // the compute warps only
  uint32_t qa[8][4];
  {
    const float4* tab = reinterpret_cast<const float4*>(smem + OFF_ROPE_ROW);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = gq + 8 * (e & 1);
        const int d = 16 * ks + 2 * t + 8 * (e >> 1);
        uint32_t val = 0;
        if (row < G) {
          const uint32_t x = *reinterpret_cast<const uint32_t*>(
              p.q + (static_cast<int64_t>(b) * p.Hq + gk * G + row) * 128 + d);
          const float4 cs = tab[d >> 2];
          const float cc = (d & 2) ? cs.z : cs.x, ss = (d & 2) ? cs.w : cs.y;
          val = rope_rotate_pair(x, cc, ss);
        }
        qa[ks][e] = val;
      }
    }
  }

  float m[2] = {-INFINITY, -INFINITY};
  float l[2] = {0.f, 0.f};
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  const float sl2 = p.scale_log2;
  const int rbase = 16 * warp;

  for (int i = 0; i < nst; ++i) {
    const uint32_t st = i % NSTAGE;
    if (!mbar_wait(full(st), (i / NSTAGE) & 1, wc)) break;
    const uint32_t kbase = sbase + st * STAGE, vbase = kbase + 2 * KHALF;
    const int nabs = n0 + i * ROWS + rbase;  // cache row of this warp's first stage row

    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    {
      const int mi = lane >> 3, rr = lane & 7;
      const int row = rbase + 8 * (mi >> 1) + rr;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int d = 16 * ks + 8 * (mi & 1);
        uint32_t b00, b01, b10, b11;
        ldmatrix_x4(kbase + (d >> 6) * KHALF + sw128_off(row, (d & 63) >> 3), b00, b01, b10, b11);
        mma_bf16_16816(sc[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b00, b01);
        mma_bf16_16816(sc[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b10, b11);
      }
    }
    // mask rows at or past len, scale into log2 units
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nabs + 8 * nt + 2 * t + (e & 1);
        sc[nt][e] = (col < len) ? sc[nt][e] * sl2 : -INFINITY;
      }
    float pr[2][4];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {  // hr 0: head row gq, hr 1: head row gq + 8
      float mx = fmaxf(fmaxf(sc[0][2 * hr], sc[0][2 * hr + 1]), fmaxf(sc[1][2 * hr], sc[1][2 * hr + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mn = fmaxf(m[hr], mx);
      const float alpha = (mn == -INFINITY) ? 1.f : ex2_approx(m[hr] - mn);
      const float mu = (mn == -INFINITY) ? 0.f : mn;
      m[hr] = mn;
      float rs = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float pv = ex2_approx(sc[nt][2 * hr + e] - mu);
          pr[nt][2 * hr + e] = pv;
          rs += pv;
        }
      l[hr] = l[hr] * alpha + rs;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][2 * hr] *= alpha;
        o[n][2 * hr + 1] *= alpha;
      }
    }
    const uint32_t a0 = pack_bf16x2(pr[0][0], pr[0][1]);
    const uint32_t a1 = pack_bf16x2(pr[0][2], pr[0][3]);
    const uint32_t a2 = pack_bf16x2(pr[1][0], pr[1][1]);
    const uint32_t a3 = pack_bf16x2(pr[1][2], pr[1][3]);

    // value rows at or past len may hold anything (NaN included): zero them so
    // that P = 0 cannot meet NaN inside the MMA.
    const bool tail = nabs + 16 > len;
    if (tail) {
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int idx = lane + 32 * x;            // 0..255: (row, half, chunk)
        const int rr = idx >> 4, hf = (idx >> 3) & 1, ch = idx & 7;
        if (nabs + rr >= len)
          *reinterpret_cast<uint4*>(smem + st * STAGE + 2 * KHALF + hf * KHALF + (rbase + rr) * 128 + ch * 16) =
              make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
    }
    {
      const int mi = lane >> 3, rr = lane & 7;
      const int row = rbase + 8 * (mi & 1) + rr;
#pragma unroll
      for (int dn2 = 0; dn2 < 8; ++dn2) {
        const int d = 16 * dn2 + 8 * (mi >> 1);
        uint32_t v0, v1, v2, v3;
        ldmatrix_x4_trans(vbase + (d >> 6) * KHALF + sw128_off(row, (d & 63) >> 3), v0, v1, v2, v3);
        mma_bf16_16816(o[2 * dn2], a0, a1, a2, a3, v0, v1);
        mma_bf16_16816(o[2 * dn2 + 1], a0, a1, a2, a3, v2, v3);
      }
    }
    if (tail) fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(st));
  }

  // ---- merge the four warps' partials (ring memory is free once all warps are here)
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    l[hr] += __shfl_xor_sync(0xffffffffu, l[hr], 1);
    l[hr] += __shfl_xor_sync(0xffffffffu, l[hr], 2);
  }
  asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
  float* cm = reinterpret_cast<float*>(smem);          // [NCW][16] running max
  float* cl = cm + NCW * 16;                           // [NCW][16] running sum
  float* co = cl + NCW * 16;                           // [NCW][16][128] partial O
  if (t == 0) {
    cm[warp * 16 + gq] = m[0];
    cm[warp * 16 + gq + 8] = m[1];
    cl[warp * 16 + gq] = l[0];
    cl[warp * 16 + gq + 8] = l[1];
  }
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const int d = 8 * n + 2 * t;
    co[(warp * 16 + gq) * 128 + d] = o[n][0];
    co[(warp * 16 + gq) * 128 + d + 1] = o[n][1];
    co[(warp * 16 + gq + 8) * 128 + d] = o[n][2];
    co[(warp * 16 + gq + 8) * 128 + d + 1] = o[n][3];
  }
  asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
  {
    const int row = threadIdx.x >> 3;          // 0..15
    const int d0 = (threadIdx.x & 7) * 16;
    if (row < G) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, cm[w * 16 + row]);
      float f[NCW], L = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        f[w] = (cm[w * 16 + row] == -INFINITY) ? 0.f : ex2_approx(cm[w * 16 + row] - M);
        L += f[w] * cl[w * 16 + row];
      }
      const float inv = 1.f / L;
      const int64_t slot = (static_cast<int64_t>(b) * p.Hq + gk * G + row) * p.nchunk + c;
      float4* dst = reinterpret_cast<float4*>(p.part_o + slot * 128 + d0);
#pragma unroll
      for (int d = 0; d < 16; d += 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
          const float* src = co + (w * 16 + row) * 128 + d0 + d;
          acc.x += f[w] * src[0];
          acc.y += f[w] * src[1];
          acc.z += f[w] * src[2];
          acc.w += f[w] * src[3];
        }
        acc.x *= inv;
        acc.y *= inv;
        acc.z *= inv;
        acc.w *= inv;
        dst[d >> 2] = acc;
      }
      if (d0 == 0) p.part_lse[slot] = M + __log2f(L);
    }
  }
}

__global__ void __launch_bounds__(128)
    decode_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                          const int32_t* __restrict__ lens, uint16_t* __restrict__ out, int Hq, int Lmax,
                          int nchunk) {
  const int bh = blockIdx.x, b = bh / Hq, d = threadIdx.x;
  const int raw = lens[b];
  if (d == 0 && bh % Hq == 0 && (raw < 0 || raw > Lmax)) raise_error(LLAMA_ATTN_DEVERR_CACHE_LEN);
  const int len = valid_len(raw, Lmax);
  const int nc = (len + CHUNK - 1) / CHUNK;
  const float* lse = part_lse + static_cast<int64_t>(bh) * nchunk;
  const float* po = part_o + static_cast<int64_t>(bh) * nchunk * 128;
  float M = -INFINITY;
  for (int c = 0; c < nc; ++c) M = fmaxf(M, lse[c]);
  float num = 0.f, den = 0.f;
  for (int c = 0; c < nc; ++c) {
    const float w = ex2_approx(lse[c] - M);
    den += w;
    num += w * po[c * 128 + d];
  }
  const float r = (nc > 0) ? num / den : 0.f;
  const __nv_bfloat16 h = __float2bfloat16_rn(r);
  out[static_cast<int64_t>(bh) * 128 + d] = *reinterpret_cast<const uint16_t*>(&h);
}

}  // namespace dec
}  // namespace la
