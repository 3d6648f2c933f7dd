// Block pattern discovery and index compaction kernels.
//
// FlashPrefill summary (zhichai.net), Method:
//   1 "Instantaneous Pattern Discovery"  -> pool_kernel (block means of Q and K)
//                                          + score_kernel (pooled scores)
//   2 "Dynamic Threshold Pruning"        -> score_kernel (alpha x row max, sink/window)
//   3 "Index Compaction -> Physical Jumps" -> score_kernel's epilogue / compact_kernel
//
// pool_kernel streams Q and K once from HBM (16-byte vector loads, float32
// accumulation); it is HBM-bound and the rest of discovery must hide behind
// it. It stores each pooled value x as three bfloat16 parts hi + mid + lo
// (24 significant bits, i.e. x itself), so that score_kernel can form the
// float32-accurate dot products q̄·k̄ on the tensor cores: with A = Ah + Am + Al
// and B = Bh + Bm + Bl, the six products Ah·Bh, Ah·Bm, Am·Bh, Am·Bm, Ah·Bl,
// Al·Bh leave out only terms below 2^-25 of |A||B| relative, and every
// bf16 x bf16 product is exact in the float32 accumulator.
//
// score_kernel: one CTA per (request, KV group, tile of 128 / G query blocks).
// The tile's score rows are (query block, head) pairs of the group; their
// pooled queries stay in shared memory while the pooled keys stream through a
// TMA ring, 128 key blocks per column tile, into double-buffered TMEM score
// tiles. Pass 1 takes every row's maximum over its causal key blocks; pass 2
// recomputes the scores, applies the threshold and the sink/window blocks,
// ORs the G heads of each query block and appends the kept blocks to the
// ascending lists (and optionally the mask words and per-head bits).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace fp {

namespace {

constexpr int kPoolThreads = 256;
// Loads per batch of a pooling thread (two batches in flight). 4 measured
// best: 8 costs occupancy (registers) and lowers the achieved bandwidth.
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

// x -> (hi, mid, lo) bf16 with hi + mid + lo == x to 24 bits: each residual
// x - hi and (x - hi) - mid is exact in float32.
__device__ __forceinline__ void split3(float x, uint16_t& h, uint16_t& m, uint16_t& l) {
  const __nv_bfloat16 bh = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(bh);
  const __nv_bfloat16 bm = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(bm);
  const __nv_bfloat16 bl = __float2bfloat16_rn(r2);
  h = __bfloat16_as_ushort(bh);
  m = __bfloat16_as_ushort(bm);
  l = __bfloat16_as_ushort(bl);
}

// Grid: first the Q work items (request, block, head chunk), then the K ones.
// Q items write the planes qpl[3][R * Nmax][Hq][D]; K items write
// kpl[3][R * Hkv][Nmax][D] (both bf16, plane 0 = hi, 1 = mid, 2 = lo).
template <bool FP8, int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(Geometry g, const uint8_t* __restrict__ q,
                                                            const uint8_t* __restrict__ k,
                                                            __nv_bfloat16* __restrict__ qpl,
                                                            __nv_bfloat16* __restrict__ kpl, int hcq, int hck,
                                                            int n_q_items) {
  constexpr int ES = FP8 ? 1 : 2;      // element size
  constexpr int EPV = 16 / ES;         // elements per 16-byte vector
  constexpr int VPH = D / EPV;         // vectors per head row
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
  const long long head_off = ((long long)h * D + e0) * ES;
  const long long row_bytes = (long long)H * D * ES;

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

  int t = t0 + p;
  // two batches of kPoolUnroll 16-byte loads: the next batch is in flight
  // while the current one is accumulated
  {
    constexpr int U = kPoolUnroll;
    const int step = U * tpi;
    uint4 xa[U], xb[U];
    auto full = [&](int tt) { return tt + (U - 1) * tpi < t1; };
    auto load = [&](uint4* x, int tt) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const long long row = row_of(tt + u * tpi);
        x[u] = row >= 0 ? ld_stream(base + row * row_bytes + head_off) : make_uint4(0, 0, 0, 0);
      }
    };
    if (full(t)) {
      load(xa, t);
      for (;;) {
        const bool nb = full(t + step);
        if (nb) load(xb, t + step);
#pragma unroll
        for (int u = 0; u < U; ++u) accumulate<FP8>(acc, xa[u]);
        t += step;
        if (!nb) break;
        const bool na = full(t + step);
        if (na) load(xa, t + step);
#pragma unroll
        for (int u = 0; u < U; ++u) accumulate<FP8>(acc, xb[u]);
        t += step;
        if (!na) break;
      }
    }
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
  uint16_t part[3][EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) split3(acc[e] * mul, part[0][e], part[1][e], part[2][e]);
  const long long plane = isK ? (long long)g.R * g.Hkv * g.Nmax * D : (long long)g.R * g.Nmax * g.Hq * D;
  __nv_bfloat16* dst = isK ? kpl + (((long long)r * g.Hkv + h) * g.Nmax + i) * D + e0
                           : qpl + (((long long)r * g.Nmax + i) * g.Hq + h) * D + e0;
#pragma unroll
  for (int pl = 0; pl < 3; ++pl) {
#pragma unroll
    for (int e = 0; e < EPV; e += 8) {
      uint4 w;
      w.x = part[pl][e] | ((uint32_t)part[pl][e + 1] << 16);
      w.y = part[pl][e + 2] | ((uint32_t)part[pl][e + 3] << 16);
      w.z = part[pl][e + 4] | ((uint32_t)part[pl][e + 5] << 16);
      w.w = part[pl][e + 6] | ((uint32_t)part[pl][e + 7] << 16);
      *reinterpret_cast<uint4*>(dst + pl * plane + e) = w;
    }
  }
}

// ---------------------------------------------------------------------------
// scoring on the tensor cores
// ---------------------------------------------------------------------------
constexpr int kScoreThreads = 192;  // warps 0-3: one score row (TMEM lane) per thread; 4: TMA; 5: MMA
constexpr int kTmaWarp = 4;
constexpr int kScoreMmaWarp = 5;
constexpr int kTile = 128 * 128;    // 128 rows x 64 bf16: one 128-byte swizzled row per score row / key block
constexpr int kScoreStages = 2;     // key ring: one stage = the three planes of one 64-wide d chunk
constexpr int kScoreBars = 1 + 2 * kScoreStages + 4 + 1;
// DC = D / 64 chunks of 64 pooled dimensions (one 128-byte swizzled row each)
template <int DC>
struct ScoreSmem {
  static constexpr int value = 1024 + 3 * DC * kTile + kScoreStages * 3 * kTile + 128 * 4 * 4 + 128 * 4 +
                               kScoreBars * 8 + 64;
};
// plane pairs of the six products, largest terms first
__constant__ int8_t kProdA[6] = {0, 0, 1, 1, 0, 2};
__constant__ int8_t kProdB[6] = {0, 1, 0, 1, 2, 0};

// AND of `ok` over the 128 epilogue threads (named barrier 1): every decision
// to stop is taken by all of them together.
__device__ __forceinline__ bool epi_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// bits e of a 32-bit word (key blocks jb + e) with lo <= jb + e < hi
__device__ __forceinline__ uint32_t bit_range(int jb, int lo, int hi) {
  const int a = max(lo - jb, 0), b = min(hi - jb, 32);
  if (a >= b) return 0u;
  const uint32_t upto = b >= 32 ? 0xFFFFFFFFu : ((1u << b) - 1u);
  return upto & ~((1u << a) - 1u);
}

template <int G, int DC>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, const Geometry g,
                 uint32_t a_bytes, uint32_t b_bytes, uint32_t* __restrict__ mask, int32_t* __restrict__ idx,
                 int32_t* __restrict__ cnt) {
  constexpr int QB = 128 / G;   // query blocks per tile
  constexpr int ROWS = QB * G;  // score rows in use
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                   // [plane][d chunk] pooled queries
  uint8_t* sB = sA + 3 * DC * kTile;                    // [stage][plane] pooled keys
  uint32_t* kw = reinterpret_cast<uint32_t*>(sB + kScoreStages * 3 * kTile);  // [row][4] keep words
  int* cbase = reinterpret_cast<int*>(kw + 128 * 4);  // [QB] list length so far
  uint64_t* bars = reinterpret_cast<uint64_t*>(cbase + 128);
  uint64_t* a_full = bars;
  uint64_t* b_full = bars + 1;
  uint64_t* b_empty = b_full + kScoreStages;
  uint64_t* s_full = b_empty + kScoreStages;  // [2]
  uint64_t* s_empty = s_full + 2;             // [2]
  uint64_t* drain = s_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kScoreBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);


  const int RH = g.R * g.Hkv;
  const int tiles = (g.Nmax + QB - 1) / QB;
  const int tile = tiles - 1 - (int)(blockIdx.x / RH);  // longest rows first
  const int rg = blockIdx.x % RH;
  const int r = rg / g.Hkv, kvh = rg % g.Hkv;
  const int i0 = tile * QB;
  const int iend = min(i0 + QB, g.Nmax);  // rows i0..iend-1 of the outputs belong to this CTA
  int qoff, qlen, kvlen;
  request_spans(g, r, qoff, qlen, kvlen);
  const int Nr = (kvlen + g.B - 1) / g.B;
  const int ifirst = (kvlen - qlen) / g.B;  // blocks before it hold no query
  const int ilast = min(iend, Nr) - 1;      // last row with keys
  const int lo_row = max(i0, ifirst);
  if (lo_row > ilast) {  // no row of this tile has a query: empty lists
    for (int x = threadIdx.x; x < iend - i0; x += kScoreThreads) {
      const long long rowi = row_index(r, kvh, i0 + x, g.Hkv, g.Nmax);
      if (cnt) cnt[rowi] = 0;
      if (mask)
        for (int w = 0; w < g.Wmax; ++w) mask[rowi * g.Wmax + w] = 0u;
    }
    return;
  }
  const int NT = ilast / 128 + 1;  // column tiles: key blocks 0..ilast
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    for (int s = 0; s < kScoreStages; ++s) {
      mbar_init(b_full + s, 1);
      mbar_init(b_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_empty + b, 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kScoreMmaWarp) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_arrive_expect_tx(a_full, 3u * DC * a_bytes);
      for (int pl = 0; pl < 3; ++pl)
        for (int c = 0; c < DC; ++c)
          tma_load_4d(sA + (pl * DC + c) * kTile, &tmQ, a_full, c * 64, kvh * G, r * g.Nmax + i0, pl);
      bool ok = true;
      int n = 0;
      for (int pass = 0; pass < 2 && ok; ++pass)
        for (int nt = 0; nt < NT && ok; ++nt)
          for (int c = 0; c < DC; ++c, ++n) {
            const int st = n % kScoreStages;
            ok = mbar_wait(b_empty + st, (uint32_t)((n / kScoreStages) & 1) ^ 1u, abort_flag, g.status,
                           FP_DEV_TIMEOUT);
            if (!ok) break;
            mbar_arrive_expect_tx(b_full + st, 3u * b_bytes);
            for (int pl = 0; pl < 3; ++pl)
              tma_load_4d(sB + (st * 3 + pl) * kTile, &tmK, b_full + st, c * 64, nt * 128, rg, pl);
          }
      // every copy this CTA issued lands before its shared memory is released,
      // also when another role gave up after this loop ended
      for (int t = n - 1; t >= 0 && t >= n - kScoreStages; --t)
        mbar_drain(b_full + t % kScoreStages, (uint32_t)((t / kScoreStages) & 1), g.status, FP_DEV_TIMEOUT);
      mbar_drain(a_full, 0u, g.status, FP_DEV_TIMEOUT);
    }
  } else if (warp == kScoreMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = instr_desc(1u, 128, 128, 0, 0);
      const uint32_t sAa = smem_u32(sA), sBa = smem_u32(sB);
      bool ok = mbar_wait(a_full, 0u, abort_flag, g.status, FP_DEV_TIMEOUT);
      tc_fence_after();
      int n = 0, q = 0;
      for (int pass = 0; pass < 2 && ok; ++pass)
        for (int nt = 0; nt < NT && ok; ++nt, ++q) {
          const int buf = q & 1;
          ok = mbar_wait(s_empty + buf, (uint32_t)((q >> 1) & 1) ^ 1u, abort_flag, g.status, FP_DEV_TIMEOUT);
          if (!ok) break;
          tc_fence_after();
          for (int c = 0; c < DC && ok; ++c, ++n) {
            const int st = n % kScoreStages;
            ok = mbar_wait(b_full + st, (uint32_t)((n / kScoreStages) & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
              for (int pr = 0; pr < 6; ++pr) {
                const uint64_t ad = smem_desc_sw128(sAa + (kProdA[pr] * DC + c) * kTile + ks * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(sBa + (st * 3 + kProdB[pr]) * kTile + ks * 32, 16, 1024);
                umma_f16_ss(tmem + buf * 128, ad, bd, idesc, (c | ks | pr) ? 1u : 0u);
              }
            }
            umma_commit(b_empty + st);
          }
          if (ok) umma_commit(s_full + buf);
        }
      // every MMA this thread issued has completed once `drain` flips
      umma_commit(drain);
      mbar_drain(drain, 0u, g.status, FP_DEV_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ epilogue: thread = score row
    const int m = threadIdx.x;
    const int ii = m / G;
    const int i = i0 + ii;
    const bool row_ok = m < ROWS && i >= lo_row && i <= ilast;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    float vmax = -INFINITY;
    int q = 0;
    bool ok = true;
    // pass 1: the row maximum over key blocks j <= i (scale > 0 commutes with max)
    for (int nt = 0; nt < NT; ++nt, ++q) {
      const int buf = q & 1;
      ok = epi_all(mbar_wait(s_full + buf, (uint32_t)((q >> 1) & 1), abort_flag, g.status, FP_DEV_TIMEOUT));
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(trow + buf * 128 + cc * 32, v);
        tmem_wait_ld();
        const int jb = nt * 128 + cc * 32;
        if (jb + 31 <= i) {
#pragma unroll
          for (int e = 0; e < 32; ++e) vmax = fmaxf(vmax, __uint_as_float(v[e]));
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (jb + e <= i) vmax = fmaxf(vmax, __uint_as_float(v[e]));
        }
      }
      tc_fence_before();
      mbar_arrive(s_empty + buf);
    }
    const float M = vmax * g.scale;
    for (int x = m; x < QB; x += 128) cbase[x] = 0;
    epi_sync();
    // pass 2: keep bits, group union, lists
    for (int nt = 0; nt < NT && ok; ++nt, ++q) {
      const int buf = q & 1;
      ok = epi_all(mbar_wait(s_full + buf, (uint32_t)((q >> 1) & 1), abort_flag, g.status, FP_DEV_TIMEOUT));
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(trow + buf * 128 + cc * 32, v);
        tmem_wait_ld();
        const int jb = nt * 128 + cc * 32;
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 32; ++e) word |= (uint32_t)(__uint_as_float(v[e]) * g.scale - M >= g.thr) << e;
        // forced sink and window blocks (kept by every head), causal j <= i
        word = (word | bit_range(jb, 0, g.Sb) | bit_range(jb, i - g.Wb + 1, i + 1)) & bit_range(jb, 0, i + 1);
        kw[m * 4 + cc] = row_ok ? word : 0u;
      }
      tc_fence_before();
      mbar_arrive(s_empty + buf);
      epi_sync();
      // one thread per (query block, word): union over the group's heads, then
      // ascending list entries after the ones of earlier column tiles
      for (int x0 = 0; x0 < QB * 4; x0 += 128) {
        const int x = x0 + m;
        const bool act = x < QB * 4;
        const int qi = x >> 2, cw = x & 3;
        const int irow = i0 + qi;
        const int wi = nt * 4 + cw;
        uint32_t word = 0;
        if (act) {
#pragma unroll
          for (int h = 0; h < G; ++h) word |= kw[(qi * G + h) * 4 + cw];
        }
        const int c = __popc(word);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o, 4);
          if (cw >= o) incl += y;
        }
        if (act && irow < g.Nmax) {
          const long long rowi = row_index(r, kvh, irow, g.Hkv, g.Nmax);
          if (mask && wi < g.Wmax) mask[rowi * g.Wmax + wi] = word;
          if (idx && word) {
            const long long lb = list_row_base(r, kvh, irow, g.Hkv, g.Nmax);
            int pos = cbase[qi] + incl - c;
            uint32_t bits = word;
            while (bits) {
              const int b = __ffs(bits) - 1;
              if (g.head_bits) {
                uint32_t hb = 0;
#pragma unroll
                for (int h = 0; h < G; ++h) hb |= ((kw[(qi * G + h) * 4 + cw] >> b) & 1u) << h;
                g.head_bits[lb + pos] = (uint8_t)hb;
              }
              idx[lb + pos++] = wi * 32 + b;
              bits &= bits - 1;
            }
          }
        }
        __syncwarp();
        if (act && cw == 3) cbase[qi] += incl;
      }
      epi_sync();
    }
    if (ok) {
      for (int x = m; x < iend - i0; x += 128) {
        const long long rowi = row_index(r, kvh, i0 + x, g.Hkv, g.Nmax);
        if (cnt) cnt[rowi] = cbase[x];
        if (mask)
          for (int w = NT * 4; w < g.Wmax; ++w) mask[rowi * g.Wmax + w] = 0u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kScoreMmaWarp) tmem_dealloc(tmem, 256);
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

template <int G, int DC>
fp_status_t launch_score_g(const Geometry& g, const __nv_bfloat16* qpl, const __nv_bfloat16* kpl, uint32_t* mask,
                           int32_t* idx, int32_t* cnt, cudaStream_t s) {
  constexpr int QB = 128 / G;
  // pooled queries: [3][R * Nmax][Hq][D], box = one 64-wide d chunk of G heads x QB blocks
  const int qb_box = QB < g.R * g.Nmax ? QB : g.R * g.Nmax;
  const int kb_box = g.Nmax < 128 ? g.Nmax : 128;
  CUtensorMap mq, mk;
  {
    const cuuint64_t row = 2 * 64 * DC;  // bytes of one pooled bf16 row
    const cuuint64_t dims[4] = {64 * DC, (cuuint64_t)g.Hq, (cuuint64_t)g.R * g.Nmax, 3};
    const cuuint64_t strides[3] = {row, (cuuint64_t)g.Hq * row, (cuuint64_t)g.R * g.Nmax * g.Hq * row};
    const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)qb_box, 1};
    if (!encode_tiled(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, qpl, dims, strides, box)) return FP_ERR_CUDA;
  }
  {
    const cuuint64_t row = 2 * 64 * DC;
    const cuuint64_t dims[4] = {64 * DC, (cuuint64_t)g.Nmax, (cuuint64_t)g.R * g.Hkv, 3};
    const cuuint64_t strides[3] = {row, (cuuint64_t)g.Nmax * row, (cuuint64_t)g.R * g.Hkv * g.Nmax * row};
    const cuuint32_t box[4] = {64, (cuuint32_t)kb_box, 1, 1};
    if (!encode_tiled(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, kpl, dims, strides, box)) return FP_ERR_CUDA;
  }
  constexpr int kSmem = ScoreSmem<DC>::value;
  cudaError_t e = cudaFuncSetAttribute(score_kernel<G, DC>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) {
    set_last_error("score smem attribute", (int)e, cudaGetErrorString(e));
    return FP_ERR_CUDA;
  }
  const unsigned grid = (unsigned)(g.R * g.Hkv * ((g.Nmax + QB - 1) / QB));
  const uint32_t a_bytes = 128u * G * qb_box, b_bytes = 128u * kb_box;
  score_kernel<G, DC><<<grid, kScoreThreads, kSmem, s>>>(mq, mk, g, a_bytes, b_bytes, mask, idx, cnt);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("score launch", (int)e, cudaGetErrorString(e));
    return FP_ERR_CUDA;
  }
  return FP_OK;
}

}  // namespace

size_t pooled_q_elems(const Geometry& g) { return (size_t)g.R * g.Nmax * g.Hq * g.d; }
size_t pooled_k_elems(const Geometry& g) { return (size_t)g.R * g.Hkv * g.Nmax * g.d; }

cudaError_t launch_pool(const Geometry& g, const void* q, const void* k, __nv_bfloat16* qpl, __nv_bfloat16* kpl,
                        cudaStream_t s) {
  const int cap = g.fp8 ? 16 : 8;  // keeps at least two tokens per iteration of 256 threads
  const int hcq = pow2_divisor(g.Hq, cap), hck = pow2_divisor(g.Hkv, cap);
  const int nq = g.R * g.Nmax * (g.Hq / hcq);
  const int nk = g.R * g.Nmax * (g.Hkv / hck);
  const uint8_t *q8 = (const uint8_t*)q, *k8 = (const uint8_t*)k;
  if (g.fp8)  // e4m3 inputs: head dim 128
    pool_kernel<true, 128><<<nq + nk, kPoolThreads, 0, s>>>(g, q8, k8, qpl, kpl, hcq, hck, nq);
  else if (g.d == 128)
    pool_kernel<false, 128><<<nq + nk, kPoolThreads, 0, s>>>(g, q8, k8, qpl, kpl, hcq, hck, nq);
  else
    pool_kernel<false, 64><<<nq + nk, kPoolThreads, 0, s>>>(g, q8, k8, qpl, kpl, hcq, hck, nq);
  return cudaGetLastError();
}

fp_status_t launch_score(const Geometry& g, const __nv_bfloat16* qpl, const __nv_bfloat16* kpl, uint32_t* mask,
                         int32_t* idx, int32_t* cnt, cudaStream_t s) {
  const bool dc2 = g.d == 128;  // pooled rows of 128 (two 64-wide chunks) or 64 dimensions
  switch (g.G) {
    case 1: return dc2 ? launch_score_g<1, 2>(g, qpl, kpl, mask, idx, cnt, s)
                  : launch_score_g<1, 1>(g, qpl, kpl, mask, idx, cnt, s);
    case 2: return dc2 ? launch_score_g<2, 2>(g, qpl, kpl, mask, idx, cnt, s)
                  : launch_score_g<2, 1>(g, qpl, kpl, mask, idx, cnt, s);
    case 3: return dc2 ? launch_score_g<3, 2>(g, qpl, kpl, mask, idx, cnt, s)
                  : launch_score_g<3, 1>(g, qpl, kpl, mask, idx, cnt, s);
    case 4: return dc2 ? launch_score_g<4, 2>(g, qpl, kpl, mask, idx, cnt, s)
                  : launch_score_g<4, 1>(g, qpl, kpl, mask, idx, cnt, s);
    case 5: return dc2 ? launch_score_g<5, 2>(g, qpl, kpl, mask, idx, cnt, s)
                  : launch_score_g<5, 1>(g, qpl, kpl, mask, idx, cnt, s);
    case 6: return dc2 ? launch_score_g<6, 2>(g, qpl, kpl, mask, idx, cnt, s)
                  : launch_score_g<6, 1>(g, qpl, kpl, mask, idx, cnt, s);
    case 7: return dc2 ? launch_score_g<7, 2>(g, qpl, kpl, mask, idx, cnt, s)
                  : launch_score_g<7, 1>(g, qpl, kpl, mask, idx, cnt, s);
    case 8: return dc2 ? launch_score_g<8, 2>(g, qpl, kpl, mask, idx, cnt, s)
                  : launch_score_g<8, 1>(g, qpl, kpl, mask, idx, cnt, s);
    case 16: return dc2 ? launch_score_g<16, 2>(g, qpl, kpl, mask, idx, cnt, s)
                  : launch_score_g<16, 1>(g, qpl, kpl, mask, idx, cnt, s);
    default: return FP_ERR_UNSUPPORTED;
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
