// Block pattern discovery and index compaction kernels.
//
// FlashPrefill summary (zhichai.net), Method:
//   1 "Instantaneous Pattern Discovery"  -> pool_kernel (block means of Q and K)
//                                          + score_kernel (pooled scores)
//   2 "Dynamic Threshold Pruning"        -> score_kernel (alpha x row max, sink/window)
//   3 "Index Compaction -> Physical Jumps" -> score_kernel's fused epilogue / compact_kernel
//
// pool_kernel streams Q and K once from HBM (16-byte vector loads, float32
// accumulation); it is HBM-bound. The pooled tensors (float32, a few MB) stay
// in L2 for score_kernel, which is FMA-bound: one CTA per (request, KV group,
// query block) row computes the G heads' scores against every causal key block
// with register blocking (4 key blocks x G heads per lane), reduces each head's
// row max, applies the threshold, ORs over the group and forces the sink and
// window blocks, then ballots the keep bits into mask words and, optionally,
// writes the compacted ascending list with a block-wide prefix sum.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.cuh"

namespace fp {

namespace {

constexpr int kPoolThreads = 256;
constexpr int kScoreThreads = 256;
// Loads in flight per pooling thread. 4 measured best: 8 costs occupancy
// (registers) and lowers the achieved bandwidth.
#ifndef FP_POOL_UNROLL
#define FP_POOL_UNROLL 4
#endif
constexpr int kPoolUnroll = FP_POOL_UNROLL;

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <bool FP8>
__device__ __forceinline__ void accumulate(float* acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if constexpr (FP8) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const __nv_fp8x2_storage_t pr = (__nv_fp8x2_storage_t)((w[q] >> (16 * hlf)) & 0xFFFFu);
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pr, __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        acc[4 * q + 2 * hlf] += f.x;
        acc[4 * q + 2 * hlf + 1] += f.y;
      }
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]));
      acc[2 * q] += f.x;
      acc[2 * q + 1] += f.y;
    }
  }
}

// Grid: first the Q work items (request, block, head chunk), then the K ones.
// Q items write qbar [R, Nmax, Hq, d]; K items write kbarT [R, Hkv, d, Npad]
// (transposed so that the scoring loads of consecutive key blocks coalesce).
template <bool FP8>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(Geometry g, const uint8_t* __restrict__ q,
                                                            const uint8_t* __restrict__ k,
                                                            float* __restrict__ qbar,
                                                            float* __restrict__ kbarT, int hcq, int hck,
                                                            int n_q_items) {
  constexpr int ES = FP8 ? 1 : 2;      // element size
  constexpr int EPV = 16 / ES;         // elements per 16-byte vector
  constexpr int VPH = 128 / EPV;       // vectors per head row (d = 128)
  __shared__ __align__(16) float red[kPoolThreads * EPV];

  int item = blockIdx.x;
  const bool isK = item >= n_q_items;
  if (isK) item -= n_q_items;
  const int H = isK ? g.Hkv : g.Hq;
  const int hc = isK ? hck : hcq;
  const int chunks = H / hc;
  const int c = item % chunks;
  const int i = (item / chunks) % g.Nmax;
  const int r = item / (chunks * g.Nmax);

  int qoff, qlen, kvlen;
  request_spans(g, r, qoff, qlen, kvlen);
  const int p0 = kvlen - qlen;  // position of the first query
  // keys: every token of the block; queries: those at positions >= p0
  const int t0 = isK ? i * g.B : max(i * g.B, p0);
  const int t1 = min(i * g.B + g.B, kvlen);
  if (t0 >= t1) return;

  const int vpt = hc * VPH;            // vectors per token row of the chunk
  const int tpi = kPoolThreads / vpt;  // tokens per iteration
  const int v = threadIdx.x % vpt;
  const int p = threadIdx.x / vpt;
  const int h = c * hc + v / VPH;
  const int e0 = (v % VPH) * EPV;
  const uint8_t* base = isK ? k : q;
  const bool paged = isK && g.page_table != nullptr;
  const long long head_off = ((long long)h * 128 + e0) * ES;
  const long long row_bytes = (long long)H * 128 * ES;

  float acc[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.f;

  auto row_of = [&](int t) -> long long {
    if (paged) {
      int pg = __ldg(g.page_table + (long long)r * g.max_pages + (t >> g.page_shift));
      if (pg < 0 || pg >= g.num_pages) {
        atomicOr(g.status, FP_DEV_BAD_PAGE);
        return -1;
      }
      return (long long)pg * g.page_size + (t & (g.page_size - 1));
    }
    return isK ? (long long)qoff + t : (long long)qoff + t - p0;
  };

  // kPoolUnroll independent 16-byte loads in flight per thread
  int t = t0 + p;
  for (; t + (kPoolUnroll - 1) * tpi < t1; t += kPoolUnroll * tpi) {
    uint4 x[kPoolUnroll];
#pragma unroll
    for (int u = 0; u < kPoolUnroll; ++u) {
      const long long row = row_of(t + u * tpi);
      x[u] = row >= 0 ? ld_stream(base + row * row_bytes + head_off) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kPoolUnroll; ++u) accumulate<FP8>(acc, x[u]);
  }
  for (; t < t1; t += tpi) {
    const long long row = row_of(t);
    if (row >= 0) accumulate<FP8>(acc, ld_stream(base + row * row_bytes + head_off));
  }

  float4* red4 = reinterpret_cast<float4*>(red);
#pragma unroll
  for (int e = 0; e < EPV; e += 4)
    red4[(threadIdx.x * EPV + e) / 4] = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
  __syncthreads();
  if (p != 0) return;
  for (int pp = 1; pp < tpi; ++pp) {
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[e] += red[((pp * vpt + v) * EPV) + e];
  }
  float mul = 1.f / (float)(t1 - t0);
  if (FP8) mul *= __ldg((isK ? g.k_scale : g.q_scale) + h);
  if (!isK) {
    float4* dst = reinterpret_cast<float4*>(qbar + (((long long)r * g.Nmax + i) * g.Hq + h) * 128 + e0);
#pragma unroll
    for (int e = 0; e < EPV; e += 4)
      dst[e / 4] = make_float4(acc[e] * mul, acc[e + 1] * mul, acc[e + 2] * mul, acc[e + 3] * mul);
  } else {
    float* dst = kbarT + (((long long)r * g.Hkv + h) * 128 + e0) * g.Npad + i;
#pragma unroll
    for (int e = 0; e < EPV; ++e) dst[(long long)e * g.Npad] = acc[e] * mul;
  }
}

// One CTA per (request r, KV group kvh, query block i); CTAs are ordered by
// descending i so that the longest rows start first.
template <int G>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(Geometry g, const float* __restrict__ qbar,
                                                              const float* __restrict__ kbarT,
                                                              uint32_t* __restrict__ mask,
                                                              int32_t* __restrict__ idx,
                                                              int32_t* __restrict__ cnt) {
  constexpr int GP = (G + 3) / 4 * 4;
  extern __shared__ __align__(16) float smem[];
  float* qsT = smem;                                           // [128][GP]
  float* sc = qsT + 128 * GP;                                  // [G][Npad]
  uint32_t* words = reinterpret_cast<uint32_t*>(sc + G * g.Npad);  // [Wmax]
  uint8_t* hbits = reinterpret_cast<uint8_t*>(words + g.Wmax);      // [Npad] per-head bits (optional)
  __shared__ float mx[G];
  __shared__ int warp_tot[kScoreThreads / 32];

  // a following programmatic-dependent launch (the attention) may start its prologue
  asm volatile("griddepcontrol.launch_dependents;");
  if (blockIdx.x == 0 && threadIdx.x == 0 && g.attn_queue) *g.attn_queue = 0;
  const int RH = g.R * g.Hkv;
  const int i = g.Nmax - 1 - (int)(blockIdx.x / RH);
  const int rg = blockIdx.x % RH;
  const int r = rg / g.Hkv, kvh = rg % g.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long rowi = row_index(r, kvh, i, g.Hkv, g.Nmax);

  int qoff, qlen, kvlen;
  request_spans(g, r, qoff, qlen, kvlen);
  const int Nr = (kvlen + g.B - 1) / g.B;
  if (i >= Nr || (i + 1) * g.B <= kvlen - qlen) {  // past the end, or no query in the block
    if (mask)
      for (int w = threadIdx.x; w < g.Wmax; w += kScoreThreads) mask[rowi * g.Wmax + w] = 0u;
    if (cnt && threadIdx.x == 0) cnt[rowi] = 0;
    return;
  }

  // pooled queries of the group's G heads, transposed to [c][head]
  const float* qsrc = qbar + (((long long)r * g.Nmax + i) * g.Hq + (long long)kvh * G) * 128;
  for (int x = threadIdx.x; x < 128 * GP; x += kScoreThreads) {
    const int hh = x % GP, cc = x / GP;
    qsT[x] = hh < G ? qsrc[hh * 128 + cc] : 0.f;
  }
  __syncthreads();

  const int n = i + 1;
  const float* kb = kbarT + ((long long)rg * 128) * g.Npad;
  // scores s[hh][j] = scale * qbar_hh . kbar_j, j = 0..i; lane owns 4 consecutive j
  for (int jb = warp * 128; jb < n; jb += 128 * (kScoreThreads / 32)) {
    const int j4 = jb + 4 * lane;
    if (j4 < n) {
      float acc[4][G];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int hh = 0; hh < G; ++hh) acc[a][hh] = 0.f;
#pragma unroll 4
      for (int cc = 0; cc < 128; ++cc) {
        const float4 kv = __ldg(reinterpret_cast<const float4*>(kb + (long long)cc * g.Npad + j4));
        const float4* qv = reinterpret_cast<const float4*>(qsT + cc * GP);
        float qq[GP];
#pragma unroll
        for (int u = 0; u < GP / 4; ++u) {
          const float4 t = qv[u];
          qq[4 * u] = t.x;
          qq[4 * u + 1] = t.y;
          qq[4 * u + 2] = t.z;
          qq[4 * u + 3] = t.w;
        }
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          acc[0][hh] = fmaf(kv.x, qq[hh], acc[0][hh]);
          acc[1][hh] = fmaf(kv.y, qq[hh], acc[1][hh]);
          acc[2][hh] = fmaf(kv.z, qq[hh], acc[2][hh]);
          acc[3][hh] = fmaf(kv.w, qq[hh], acc[3][hh]);
        }
      }
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
        *reinterpret_cast<float4*>(sc + hh * g.Npad + j4) =
            make_float4(acc[0][hh] * g.scale, acc[1][hh] * g.scale, acc[2][hh] * g.scale, acc[3][hh] * g.scale);
    }
  }
  __syncthreads();

  // each head's row max over j <= i
  for (int hh = warp; hh < G; hh += kScoreThreads / 32) {
    float m = -INFINITY;
    for (int j = lane; j < n; j += 32) m = fmaxf(m, sc[hh * g.Npad + j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) mx[hh] = m;
  }
  __syncthreads();

  // keep bits: threshold per head, union over the group, forced sink/window
  // (a forced block counts as kept by every head of the group)
  for (int w = warp; w < g.Wmax; w += kScoreThreads / 32) {
    const int j = 32 * w + lane;
    uint32_t hb = 0;
    if (j < n) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh) hb |= (uint32_t)(sc[hh * g.Npad + j] - mx[hh] >= g.thr) << hh;
      if ((j < g.Sb) || (i - j < g.Wb)) hb = (1u << G) - 1u;
      if (g.head_bits) hbits[j] = (uint8_t)hb;
    }
    const bool keep = hb != 0;
    const uint32_t bits = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) {
      words[w] = bits;
      if (mask) mask[rowi * g.Wmax + w] = bits;
    }
  }
  if (idx == nullptr) return;
  __syncthreads();

  // fused compaction: block-wide exclusive prefix of the words' popcounts
  const int nw = (n + 31) / 32;  // <= Wmax <= kScoreThreads (checked on the host)
  const uint32_t mine = threadIdx.x < nw ? words[threadIdx.x] : 0u;
  const int c = __popc(mine);
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kScoreThreads / 32; ++w) {
    const int t = warp_tot[w];
    before += w < warp ? t : 0;
    total += t;
  }
  int pos = before + incl - c;
  const long long base = list_row_base(r, kvh, i, g.Hkv, g.Nmax);
  int32_t* dst = idx + base;
  uint8_t* hdst = g.head_bits ? g.head_bits + base : nullptr;
  uint32_t bits = mine;
  while (bits) {
    const int b = __ffs(bits) - 1;
    const int j = 32 * (int)threadIdx.x + b;
    if (hdst) hdst[pos] = hbits[j];
    dst[pos++] = j;
    bits &= bits - 1;
  }
  if (threadIdx.x == 0) cnt[rowi] = total;
}

// One warp per mask row: popcount, warp prefix sum, ordered writes. Bits above
// the diagonal (j > i) are ignored so a row never exceeds its capacity i + 1.
__global__ void __launch_bounds__(256) compact_kernel(Geometry g, const uint32_t* __restrict__ mask,
                                                      int32_t* __restrict__ idx, int32_t* __restrict__ cnt) {
  const long long rows = (long long)g.R * g.Hkv * g.Nmax;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int i = (int)(row % g.Nmax);
  const long long rk = row / g.Nmax;
  const int per = (g.Wmax + 31) / 32;
  const int w0 = lane * per;
  int c = 0;
  for (int w = w0; w < min(w0 + per, g.Wmax); ++w) {
    uint32_t x = mask[row * g.Wmax + w];
    const int lo = 32 * w;
    if (lo > i) x = 0u;
    else if (i - lo < 31) x &= (2u << (i - lo)) - 1u;
    c += __popc(x);
  }
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int pos = incl - c;
  int32_t* dst = idx + rk * ((long long)g.Nmax * (g.Nmax + 1) / 2) + (long long)i * (i + 1) / 2;
  for (int w = w0; w < min(w0 + per, g.Wmax); ++w) {
    uint32_t x = mask[row * g.Wmax + w];
    const int lo = 32 * w;
    if (lo > i) x = 0u;
    else if (i - lo < 31) x &= (2u << (i - lo)) - 1u;
    while (x) {
      const int b = __ffs(x) - 1;
      dst[pos++] = lo + b;
      x &= x - 1;
    }
  }
  if (lane == 31) cnt[row] = incl;
}

int pow2_divisor(int H, int cap) {
  int hc = 1;
  while (hc * 2 <= cap && H % (hc * 2) == 0) hc *= 2;
  return hc;
}

template <int G>
cudaError_t launch_score_g(const Geometry& g, const float* qbar, const float* kbarT, uint32_t* mask,
                           int32_t* idx, int32_t* cnt, cudaStream_t s) {
  const size_t smem = score_smem_bytes(g);
  cudaError_t e = cudaFuncSetAttribute(score_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(g.R * g.Hkv * g.Nmax);
  score_kernel<G><<<grid, kScoreThreads, smem, s>>>(g, qbar, kbarT, mask, idx, cnt);
  return cudaGetLastError();
}

}  // namespace

size_t score_smem_bytes(const Geometry& g) {
  const int GP = (g.G + 3) / 4 * 4;
  return (size_t)(128 * GP + g.G * g.Npad) * sizeof(float) + (size_t)g.Wmax * sizeof(uint32_t) + (size_t)g.Npad;
}

cudaError_t launch_pool(const Geometry& g, const void* q, const void* k, float* qbar, float* kbarT,
                        cudaStream_t s) {
  const int cap = g.fp8 ? 16 : 8;  // keeps at least two tokens per iteration of 256 threads
  const int hcq = pow2_divisor(g.Hq, cap), hck = pow2_divisor(g.Hkv, cap);
  const int nq = g.R * g.Nmax * (g.Hq / hcq);
  const int nk = g.R * g.Nmax * (g.Hkv / hck);
  if (g.fp8)
    pool_kernel<true><<<nq + nk, kPoolThreads, 0, s>>>(g, (const uint8_t*)q, (const uint8_t*)k, qbar, kbarT,
                                                       hcq, hck, nq);
  else
    pool_kernel<false><<<nq + nk, kPoolThreads, 0, s>>>(g, (const uint8_t*)q, (const uint8_t*)k, qbar, kbarT,
                                                        hcq, hck, nq);
  return cudaGetLastError();
}

cudaError_t launch_score(const Geometry& g, const float* qbar, const float* kbarT, uint32_t* mask,
                         int32_t* idx, int32_t* cnt, cudaStream_t s) {
  switch (g.G) {
    case 1: return launch_score_g<1>(g, qbar, kbarT, mask, idx, cnt, s);
    case 2: return launch_score_g<2>(g, qbar, kbarT, mask, idx, cnt, s);
    case 3: return launch_score_g<3>(g, qbar, kbarT, mask, idx, cnt, s);
    case 4: return launch_score_g<4>(g, qbar, kbarT, mask, idx, cnt, s);
    case 5: return launch_score_g<5>(g, qbar, kbarT, mask, idx, cnt, s);
    case 6: return launch_score_g<6>(g, qbar, kbarT, mask, idx, cnt, s);
    case 7: return launch_score_g<7>(g, qbar, kbarT, mask, idx, cnt, s);
    case 8: return launch_score_g<8>(g, qbar, kbarT, mask, idx, cnt, s);
    case 16: return launch_score_g<16>(g, qbar, kbarT, mask, idx, cnt, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_compact(const Geometry& g, const uint32_t* mask, int32_t* idx, int32_t* cnt,
                           cudaStream_t s) {
  const long long rows = (long long)g.R * g.Hkv * g.Nmax;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  compact_kernel<<<grid, 256, 0, s>>>(g, mask, idx, cnt);
  return cudaGetLastError();
}

}  // namespace fp
