// qkv_fp8.cuh -- FP8 (E4M3) QKV projection with RoPE in the epilogue, and the
// per-tensor dynamic quantizer that feeds it.
//
// Method ("Llama 3.1 Architecture: Dense Scaling to 405B and 128K Context",
// "FP8 Quantization: Fitting 405B on an 8xH100 Node"): the attention QKV
// projection runs in E4M3 with one dynamic scale per tensor,
// X_fp8 = clip(round(X / s_X), -448, 448), W_fp8 likewise, and
// Y = (s_X s_W) (X_fp8 W_fp8). Here s = amax(|X|) / 448, round is
// round-to-nearest-even onto the E4M3 grid, and the clip is the conversion's
// saturation. The projection's query and key heads are then rotated by RoPE
// at each token's document position, so the attention reads them ready.
#pragma once

#include "ptx.cuh"

namespace la {
namespace q8 {

constexpr float kE4M3Max = 448.f;

// ---------------------------------------------------------------- quantizer

// amax of |x| over n_vec * 8 bf16 values, as float bits max-reduced with
// atomicMax (non-negative floats order like unsigned ints). *amax_bits is zero
// at launch.
__global__ void amax_bf16_kernel(const uint4* __restrict__ x, int64_t n_vec, unsigned int* __restrict__ amax_bits) {
  float m = 0.f;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // four independent 16-byte loads in flight per thread
  for (int64_t i0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i0 < n_vec; i0 += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * stride;
      v[u] = i < n_vec ? x[i] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 a = unpack_bf16x2(v[u].x), b = unpack_bf16x2(v[u].y), c = unpack_bf16x2(v[u].z),
                   d = unpack_bf16x2(v[u].w);
      m = fmaxf(m, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(b.x), fabsf(b.y))));
      m = fmaxf(m, fmaxf(fmaxf(fabsf(c.x), fabsf(c.y)), fmaxf(fabsf(d.x), fabsf(d.y))));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float s_m[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_m[warp] = m;
  __syncthreads();
  if (warp == 0) {
    m = lane < static_cast<int>(blockDim.x >> 5) ? s_m[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0 && m > 0.f) atomicMax(amax_bits, __float_as_uint(m));
  }
}

// The per-tensor scale s = amax / 448 (1 for an all-zero tensor).
__device__ __forceinline__ float scale_of(unsigned int amax_bits) {
  const float a = __uint_as_float(amax_bits);
  return a > 0.f ? __fdiv_rn(a, kE4M3Max) : 1.f;
}

// y = E4M3(x / s), s = scale_of(*amax_bits), written to *scale_out too.
// Eight values per thread step; the quotient is an IEEE float32 division.
__global__ void quantize_e4m3_kernel(const uint4* __restrict__ x, int64_t n_vec,
                                     const unsigned int* __restrict__ amax_bits, uint2* __restrict__ y,
                                     float* __restrict__ scale_out) {
  const float s = scale_of(*amax_bits);
  if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = s;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i0 < n_vec; i0 += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * stride;
      v[u] = i < n_vec ? x[i] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * stride;
      if (i >= n_vec) break;
      const float2 a = unpack_bf16x2(v[u].x), b = unpack_bf16x2(v[u].y), c = unpack_bf16x2(v[u].z),
                   d = unpack_bf16x2(v[u].w);
      const uint32_t lo = e4m3x2(__fdiv_rn(a.x, s), __fdiv_rn(a.y, s)) |
                          (e4m3x2(__fdiv_rn(b.x, s), __fdiv_rn(b.y, s)) << 16);
      const uint32_t hi = e4m3x2(__fdiv_rn(c.x, s), __fdiv_rn(c.y, s)) |
                          (e4m3x2(__fdiv_rn(d.x, s), __fdiv_rn(d.y, s)) << 16);
      y[i] = make_uint2(lo, hi);
    }
  }
}

// ---------------------------------------------------------------- GEMM + RoPE

// Tile: 128 tokens x 256 output features (two heads of 128), K in steps of
// 128 bytes (one 128-byte swizzle row of E4M3). tcgen05.mma M128 N256 K32,
// four per K step. Four-stage TMA ring, two TMEM accumulators (2 x 256
// columns) so a tile's epilogue overlaps the next tile's MMAs.
constexpr int BM = 128, BN = 256, BK = 128;
constexpr int NSTAGE = 4;
constexpr int A_BYTES = BM * BK;                    // 16 KB
constexpr int B_BYTES = BN * BK;                    // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;      // 48 KB
constexpr int OFF_OUT = NSTAGE * STAGE_BYTES;       // epilogue staging: one head, 128 x 128 bf16
constexpr int OUT_HALF = 16384;                     // 64 columns x 128 rows, 128-byte swizzle
constexpr int OFF_BAR = OFF_OUT + 2 * OUT_HALF;
constexpr int SMEM_USED = OFF_BAR + 256;
constexpr int SMEM_ALLOC = SMEM_USED + 1024;        // slack to align the base to 1024 bytes
static_assert(SMEM_ALLOC <= 232448, "shared memory per block");
constexpr int NTHREADS = 256;                       // warp 0 TMA, warp 1 MMA, warps 4-7 epilogue
constexpr uint32_t TMEM_COLS = 512;

enum : int { B_FULL = 0, B_EMPTY = B_FULL + NSTAGE, B_ACC_FULL = B_EMPTY + NSTAGE, B_ACC_EMPTY = B_ACC_FULL + 2,
             B_EPI = B_ACC_EMPTY + 2, B_DRAIN, N_BARS };
static_assert(N_BARS * 8 + 8 <= 256, "barrier area");

struct Params {
  int M, K, N;               // tokens, model width (bytes per X row), output features (Hq + 2 Hkv) * 128
  int Hq, Hkv, S;            // heads; tokens per batch row (positions restart per row and per document)
  int n_mt, n_nt, n_kb;      // tiles along M, N and K steps
  const int32_t* doc_start;  // [M] row-local document start, or null
  const float4* rope_tab;    // (cos, sin) of 64 pairs per position, as float4 = 2 pairs
  const float* s_x;          // device scales of X and W
  const float* s_w;
  unsigned int epoch;
};

__global__ void __launch_bounds__(NTHREADS, 1)
    qkv_fp8_rope_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 8 * N_BARS);
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtx wc{p.epoch};
  const int n_tiles = p.n_mt * p.n_nt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(B_ACC_FULL + a), 1);
      mbar_init(bar(B_ACC_EMPTY + a), 128);
    }
    mbar_init(bar(B_EPI), 128);
    mbar_init(bar(B_DRAIN), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const int mt = t / p.n_nt, nt = t % p.n_nt;
        for (int kb = 0; kb < p.n_kb; ++kb, ++it) {
          const uint32_t st = it % NSTAGE, use = it / NSTAGE;
          if (use > 0 && !mbar_wait(bar(B_EMPTY + st), (use - 1) & 1, wc)) {
            ok = false;
            break;
          }
          const uint32_t dst = sbase + st * STAGE_BYTES;
          mbar_arrive_expect_tx(bar(B_FULL + st), STAGE_BYTES);
          tma_load_2d(dst, &tm_x, bar(B_FULL + st), kb * BK, mt * BM);
          tma_load_2d(dst + A_BYTES, &tm_w, bar(B_FULL + st), kb * BK, nt * BN);
        }
      }
      // every issued load has landed before the CTA may exit
      for (uint32_t st = 0; st < NSTAGE; ++st)
        if (it > st) mbar_wait(bar(B_FULL + st), ((it - 1 - st) / NSTAGE) & 1, wc);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_e4m3_f32(BM, BN);
      uint32_t it = 0, acc_i = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++acc_i) {
        const uint32_t acc = acc_i & 1, use = acc_i >> 1;
        if (use > 0 && !mbar_wait(bar(B_ACC_EMPTY + acc), (use - 1) & 1, wc)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = 0; kb < p.n_kb; ++kb, ++it) {
          const uint32_t st = it % NSTAGE;
          if (!mbar_wait(bar(B_FULL + st), (it / NSTAGE) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = umma_desc_sw128(sbase + st * STAGE_BYTES, 16, 1024);
          const uint64_t db = umma_desc_sw128(sbase + st * STAGE_BYTES + A_BYTES, 16, 1024);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)  // K = 32 E4M3 = 32 bytes per MMA: +2 in the >>4 address field
            tc_mma_ss_f8(d, da + 2u * k, db + 2u * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          tc_commit(bar(B_EMPTY + st));
        }
        if (ok) tc_commit(bar(B_ACC_FULL + acc));
      }
      tc_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, wc);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 4;
    const int r = ew * 32 + lane;                 // tile row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(ew * 32) << 16;
    uint8_t* out_stage = smem + OFF_OUT;
    const int n_heads = p.Hq + 2 * p.Hkv;
    // bounded barrier of the 128 epilogue threads (an mbarrier, so a wait that
    // runs out returns instead of hanging)
    uint32_t n_sync = 0;
    auto epi_sync = [&]() -> bool {
      mbar_arrive(bar(B_EPI));
      return mbar_wait(bar(B_EPI), (n_sync++) & 1, wc);
    };
    bool ok = true;
    uint32_t acc_i = 0;
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++acc_i) {
      const int mt = t / p.n_nt, nt = t % p.n_nt;
      const uint32_t acc = acc_i & 1, use = acc_i >> 1;
      if (!mbar_wait(bar(B_ACC_FULL + acc), use & 1, wc)) break;
      tc_fence_after();
      const float scale = __ldg(p.s_x) * __ldg(p.s_w);
      const int m = mt * BM + r;
      int pos = 0;
      if (m < p.M) pos = m % p.S - (p.doc_start ? p.doc_start[m] : 0);
      const float4* tab = p.rope_tab + static_cast<int64_t>(pos) * 32;
      for (int h = 0; h < 2; ++h) {
        const int head = nt * 2 + h;  // global head over [Q heads | K heads | V heads]
        if (head >= n_heads) break;   // the same for every thread of the tile
        const bool rotate = head < p.Hq + p.Hkv;
        // the staging buffer is free once the previous store has read it
        if (r == 0) tma_store_wait_read0();
        if (!(ok = epi_sync())) break;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + acc * BN + h * 128 + c * 32, v);
          tc_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float x0 = __uint_as_float(v[2 * j]) * scale, x1 = __uint_as_float(v[2 * j + 1]) * scale;
            if (rotate) {
              const float4 cs = __ldg(tab + c * 8 + (j >> 1));
              const float cj = (j & 1) ? cs.z : cs.x, sj = (j & 1) ? cs.w : cs.y;
              const float y0 = x0 * cj - x1 * sj, y1 = x0 * sj + x1 * cj;
              x0 = y0;
              x1 = y1;
            }
            pk[j] = pack_bf16x2(x0, x1);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int ch = c * 4 + u;  // 16-byte chunk of the 256-byte head row
            *reinterpret_cast<uint4*>(out_stage + (ch >> 3) * OUT_HALF + sw128_off(r, ch & 7)) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          }
        }
        fence_proxy_async_smem();
        if (!(ok = epi_sync())) break;
        if (r == 0) {
          const CUtensorMap* tm = head < p.Hq ? &tm_q : (head < p.Hq + p.Hkv ? &tm_k : &tm_v);
          const int hh = head < p.Hq ? head : (head < p.Hq + p.Hkv ? head - p.Hq : head - p.Hq - p.Hkv);
          tma_store_2d(tm, smem_addr(out_stage), hh * 128, mt * BM);
          tma_store_2d(tm, smem_addr(out_stage + OUT_HALF), hh * 128 + 64, mt * BM);
          tma_store_commit();
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_ACC_EMPTY + acc));
    }
    if (r == 0) tma_store_wait0();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace q8
}  // namespace la
