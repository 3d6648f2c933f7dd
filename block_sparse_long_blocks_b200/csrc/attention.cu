// Block-sparse causal prefill attention over compacted KV-block lists, sm_100a.
//
// "FlashPrefill V2" abstract: the sparse operator uses PackGQA memory access,
// warp specialisation and ping-pong pipelining, supports FP8, paged KV and
// continuous batching. FlashPrefill summary, Method 3: the inner loop visits
// only the listed blocks ("physical jumps").
//
// Work unit = (request r, KV group kvh, query block i, M-tile pair). PackGQA:
// the rows of an M-tile are (token, head) pairs of one KV group, token-major
// (row = t * G + h), Tm tokens x G heads with Tm the largest power of two such
// that Tm * G <= 128 and Tm <= B / 2, so every K/V tile a CTA loads serves all
// G heads. A CTA owns two M-tiles (ping-pong) and walks row (r, kvh, i)'s list.
//
// Roles (384 threads, one persistent CTA per SM):
//   warps 0-3  softmax warpgroup for M-tile 0 (one thread per row)
//   warps 4-7  softmax warpgroup for M-tile 1
//   warp 8     TMA producer: Q tiles, then K[idx[n]] and V[idx[n]] into rings
//   warp 9     MMA issuer (one thread): S = Q K^T into TMEM, O += P V with P
//              read from TMEM (aliasing S), accumulators in TMEM
//   warps 10-11 e4m3 inputs: widen each V tile to f16 in shared memory (exact)
//              for the PV product; bf16 inputs: idle (they complete the third
//              warpgroup for the register split)
// Operand types: S = Q K^T on the input type (bf16, or e4m3 at twice the
// tensor rate); P and V for O += P V are 16-bit (bf16, or f16 for e4m3
// inputs: f16 keeps P to 2^-11 relative, where an e4m3 P would lose 2^-4).
// Order of MMAs per visit n (ping-pong): PV0(n), S0(n+1), PV1(n), S1(n+1), so
// one warpgroup's softmax overlaps the other tile's MMAs.
// Softmax: online, base-2, with the running reference max raised only when the
// tile max exceeds it by more than a threshold (64 for bf16 P, 15 for f16 P;
// then O and l are rescaled in place).
// Every wait is time-bounded; on expiry the CTA records FP_DEV_TIMEOUT, drains
// its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <climits>
#include <cstdio>

#include "internal.cuh"
#include "sm100.cuh"

namespace fp {

namespace {

constexpr int kThreads = 384;  // 3 warpgroups
constexpr int kUnitRing = 4;                // work units handed from the producer to the other roles
// the MMA thread + both softmax warpgroups (+ the two V-converter warps for e4m3)
template <bool FP8>
struct UnitConsumers {
  static constexpr int value = 1 + 256 + (FP8 ? 64 : 0);
};
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kConvertWarp = 10;  // warps 10-11 (e4m3 inputs)
// Launched at 168 registers/thread (384 x 168 = 64512). The softmax warpgroups
// then raise their limit and the producer/MMA warpgroup lowers its own:
// 2 x 128 x 200 + 128 x 104 = 64512 <= 64512, and per SM sub-partition (three
// warps each) 2 x 32 x 200 + 32 x 104 = 16128 <= 16384. (At 96 the MMA
// issuer's loop spills.)
constexpr uint32_t kSoftmaxRegs = 200;
constexpr uint32_t kControlRegs = 104;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * 168, "register split exceeds the launch");
static_assert(2 * 32 * kSoftmaxRegs + 32 * kControlRegs <= 16384, "register split exceeds an SM sub-partition");
// The reference max is raised only when a tile's max exceeds it by more than
// this (log2 units); P is then at most 2^threshold.
// bf16 P, the float32 row sum and the float32 TMEM accumulators have float32's
// exponent range: with 2^64 per weight, 2^18 keys and |v| < 2^4 every sum stays
// below 2^86, so a rescale (a TMEM round trip of the O row) is needed only on
// jumps of the row max by more than 64 (a factor 1.8e19).
// f16 P (e4m3 inputs) must stay below 65504: threshold 15.
#ifndef FP_RESCALE_LOG2_BF16
#define FP_RESCALE_LOG2_BF16 64
#endif
template <bool FP8>
struct RescaleThreshold {
  static constexpr float value = FP8 ? 15.0f : (float)FP_RESCALE_LOG2_BF16;
};
// On a rescale the reference max is set this far below the new row max. For
// f16 P this places the running max at P = 2^8 (P stays <= 2^15 because the
// threshold still bounds the reference gap at 15) and moves f16's subnormal
// floor (2^-24) a further 2^8 below it; bf16 P has float32's range and needs
// no offset.
#ifndef FP_F16P_MAX_OFFSET
#define FP_F16P_MAX_OFFSET 8
#endif
template <bool FP8>
struct MaxOffset {
  static constexpr float value = FP8 ? (float)FP_F16P_MAX_OFFSET : 0.0f;
};
static_assert(FP_F16P_MAX_OFFSET <= 15, "f16 P would exceed 2^15");
// Shared memory for the Q tiles and the K/V rings (the opt-in maximum per CTA is 227 KB).
#ifndef FP_SMEM_BUDGET_KB
#define FP_SMEM_BUDGET_KB 200
#endif
constexpr int kSmemBudget = FP_SMEM_BUDGET_KB * 1024;

// 2^x with the MUFU.EX2 instruction (flush-to-zero, ~2 ulp); 2^-inf = +0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- packed float32x2 arithmetic (one instruction for two lanes' worth of work)
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// One pair of softmax weights 2^(s*sl2 - m) on MUFU.EX2, after a scale-and-subtract
// (packed float32x2 FMA when FP_PACKED_FMA is set, a compile-time tuning knob).
#ifndef FP_PACKED_FMA
#define FP_PACKED_FMA 1
#endif
__device__ __forceinline__ void exp2_pair(float s0, float s1, float sl2, float m_ref, uint64_t sl2x2, uint64_t negm2,
                                          float& p0, float& p1) {
  if (FP_PACKED_FMA) {
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(s0, s1), sl2x2, negm2), x0, x1);
    p0 = fast_exp2(x0);
    p1 = fast_exp2(x1);
  } else {
    p0 = fast_exp2(fmaf(s0, sl2, m_ref == -INFINITY ? 0.f : -m_ref));
    p1 = fast_exp2(fmaf(s1, sl2, m_ref == -INFINITY ? 0.f : -m_ref));
  }
}

// A pair of softmax weights as the PV product's 16-bit A operand (x0 in the
// low half): f16 for e4m3 inputs, bf16 otherwise; round to nearest.
template <bool F16>
__device__ __forceinline__ uint32_t pack_p2(float x0, float x1) {
  uint32_t u;
  if constexpr (F16) {
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(x1), "f"(x0));
  } else {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(x1), "f"(x0));
  }
  return u;
}

// e4m3 pair -> f16 pair (exact: every e4m3 value is an f16 value)
__device__ __forceinline__ uint32_t widen_e4m3x2(uint32_t two_bytes) {
  uint32_t u;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(u) : "h"((unsigned short)two_bytes));
  return u;
}

// e4m3 V tile [BLK keys][128 d] as TMA wrote it (128-byte rows, 128-byte
// swizzle: 16-byte granule p of row r sits at position p ^ (r & 7)) -> f16 tile
// in the layout TMA gives a bf16 V tile: two chunks of 64 d-elements, each
// [BLK keys][128 bytes] with the same swizzle. Thread ct of `nthreads` widens
// granules ct, ct + nthreads, ...
template <int BLK>
__device__ __forceinline__ void widen_v_tile(const uint8_t* src, uint8_t* dst, int ct, int nthreads) {
#pragma unroll 4
  for (int q = ct; q < BLK * 8; q += nthreads) {
    const int key = q >> 3, g8 = q & 7, sw = key & 7;
    const uint4 w = *reinterpret_cast<const uint4*>(src + key * 128 + ((g8 ^ sw) << 4));
    const uint4 lo = make_uint4(widen_e4m3x2(w.x), widen_e4m3x2(w.x >> 16), widen_e4m3x2(w.y),
                                widen_e4m3x2(w.y >> 16));  // d = 16 g8 + 0..7
    const uint4 hi = make_uint4(widen_e4m3x2(w.z), widen_e4m3x2(w.z >> 16), widen_e4m3x2(w.w),
                                widen_e4m3x2(w.w >> 16));  // d = 16 g8 + 8..15
    uint8_t* row = dst + (g8 >> 2) * (BLK * 128) + key * 128;
    const int p = 2 * (g8 & 3);
    *reinterpret_cast<uint4*>(row + ((p ^ sw) << 4)) = lo;
    *reinterpret_cast<uint4*>(row + (((p + 1) ^ sw) << 4)) = hi;
  }
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// acc_lo += float(low half of u); acc_hi += float(high half of u), u holding
// two f16 (F16) or two bf16 values
template <bool F16>
__device__ __forceinline__ void add_p2(float& acc_lo, float& acc_hi, uint32_t u) {
  if constexpr (F16) {
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.f16 %0, lo, %0;\n\tadd.rn.f32.f16 %1, hi, %1;\n\t}"
        : "+f"(acc_lo), "+f"(acc_hi)
        : "r"(u));
  } else {
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
        : "+f"(acc_lo), "+f"(acc_hi)
        : "r"(u));
  }
}

struct AttnArgs {
  Geometry g;
  int Tm;       // tokens per M-tile
  int rows;     // Tm * G rows in use per M-tile
  int nPairs;   // M-tile pairs per query block
  long long num_units;
  long long T;  // rows of Q / O (R*L contiguous, total_tokens varlen)
  float scale_log2;
  const int32_t* idx;
  const int32_t* cnt;
  __nv_bfloat16* o;
  float* lse;
  int* queue;          // device work-queue counter (zeroed before launch) or nullptr: static schedule
  const int* order;    // with a queue: the units in claim order (longest lists first)
};

template <bool FP8, int BLK, int D>
struct Cfg {
  static constexpr int ES = FP8 ? 1 : 2;                  // bytes per Q / K element
  static constexpr int ROW = D * ES;                      // bytes of one Q / K row
  static constexpr int DCH = ROW / 128;                   // 128-byte chunks along d of Q, K (and loaded V)
  static constexpr int CH_ELEMS = 128 / ES;               // elements per chunk
  static constexpr int Q_TILE = DCH * 128 * 128;          // bytes per 128-row M-tile
  static constexpr int KV_CHUNK = BLK * 128;              // bytes per 128-byte-wide chunk of a K/V tile
  static constexpr int K_TILE = DCH * KV_CHUNK;           // K tile (QK operand B)
  static constexpr int V_TILE = (D / 64) * KV_CHUNK;      // 16-bit V tile (PV operand B, 64 d per chunk)
  static constexpr int V8_TILE = FP8 ? DCH * KV_CHUNK : 0;  // e4m3 V tile as loaded
  static_assert(ROW % 128 == 0 && (D == 64 || D == 128), "head dim 64 (16-bit inputs) or 128");
  static_assert(!FP8 || D == 128, "e4m3 inputs need 128-byte rows: head dim 128");
  // Ring depths within the budget. bf16: K and V tiles have one size; an odd
  // slot goes to K, whose tile is consumed about one visit before the V tile
  // of the same block. e4m3: two f16 V slots, the rest shared by the e4m3 K
  // and V rings.
  static constexpr int REST = kSmemBudget - 2 * Q_TILE;
  static constexpr int TILES_RAW = REST / K_TILE;
  static constexpr int TILES = TILES_RAW > 8 ? 8 : TILES_RAW;
  static constexpr int N8 = FP8 ? (REST - 2 * V_TILE) / K_TILE : 0;
  static constexpr int V_STAGES = FP8 ? 2 : TILES / 2;
  static constexpr int K_STAGES = FP8 ? ((N8 + 1) / 2 > 4 ? 4 : (N8 + 1) / 2) : TILES - V_STAGES;
  static constexpr int V8_STAGES = FP8 ? (N8 / 2 > 4 ? 4 : N8 / 2) : 0;
  static constexpr int QK_STEPS = ROW / 32;               // K = 32 bytes per MMA: 8 (bf16) / 4 (e4m3) at d = 128
  static constexpr int PV_KEYS = 16;                      // keys per 16-bit PV MMA
  static constexpr int PV_STEPS = BLK / PV_KEYS;
  static constexpr int NUM_BARS = 2 + 2 * (K_STAGES + V_STAGES + V8_STAGES) + 8 + 1 + 2 * kUnitRing;
  static constexpr int SMEM_USED = 1024 + 2 * Q_TILE + K_STAGES * K_TILE + V_STAGES * V_TILE +
                                   V8_STAGES * V8_TILE + NUM_BARS * 8 + 16 + 4 * kUnitRing;
  // more than half of the SM's shared memory: one CTA per SM, so the CTA's
  // 512-column TMEM allocation never waits for a co-resident CTA
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static_assert(V_STAGES >= 2 && K_STAGES >= 2 && (!FP8 || V8_STAGES >= 2), "shared memory budget too small");
  static_assert(SMEM <= 227 * 1024, "beyond the per-CTA shared memory limit");
};

// Work units reach the roles either by a static stride over the persistent
// grid or, with a device queue, in claim order: the producer claims the next
// position (atomicAdd on the queue), looks the unit up in the longest-first
// order and passes it to the MMA and softmax roles through a small ring in
// shared memory guarded by full/empty mbarriers.
struct UnitIter {
  int* queue;
  const int* order;
  int* ring;
  uint64_t* full;
  uint64_t* empty;
  volatile int* abort;
  unsigned* status;
  bool producer;
  bool warp;  // consumer called by whole warps (the softmax roles)
  long long num_units;
  long long u;
  int n;

  __device__ __forceinline__ long long step(bool first, bool& ok) {
    if (queue == nullptr) {
      u = first ? (long long)blockIdx.x : u + gridDim.x;
      return u;
    }
    const int slot = n % kUnitRing;
    const uint32_t ph = (uint32_t)((n / kUnitRing) & 1);
    ++n;
    if (producer) {
      if (!mbar_wait(empty + slot, ph ^ 1u, abort, status, FP_DEV_TIMEOUT)) {
        ok = false;
        return LLONG_MAX;
      }
      int v = atomicAdd(queue, 1);
      if (v < num_units) v = __ldg(order + v);
      ring[slot] = v;
      mbar_arrive(full + slot);
      return v;
    }
    const bool got = warp ? mbar_wait<true>(full + slot, ph, abort, status, FP_DEV_TIMEOUT)
                          : mbar_wait<false>(full + slot, ph, abort, status, FP_DEV_TIMEOUT);
    if (!got) {
      ok = false;
      return LLONG_MAX;
    }
    const int v = ring[slot];
    mbar_arrive(empty + slot);
    return v;
  }
};

struct Unit {
  int r, kvh, i, pair;
  int off;    // first query row of the request
  int len;    // KV length (positions 0..len-1)
  int p0;     // position of the request's first query
  int count;
  long long lbase, rowi;
};

__device__ __forceinline__ bool decode_unit(long long u, const AttnArgs& a, Unit& U) {
  const Geometry& g = a.g;
  const long long per_i = (long long)g.R * g.Hkv * a.nPairs;
  U.i = g.Nmax - 1 - (int)(u / per_i);
  long long rem = u % per_i;
  U.pair = (int)(rem % a.nPairs);
  rem /= a.nPairs;
  U.kvh = (int)(rem % g.Hkv);
  U.r = (int)(rem / g.Hkv);
  int qlen;
  request_spans(g, U.r, U.off, qlen, U.len);
  U.p0 = U.len - qlen;
  // query positions of this pair of M-tiles, clipped to the request's queries
  const int lo = U.i * g.B + U.pair * 2 * a.Tm;
  const int hi = min(lo + 2 * a.Tm, min((U.i + 1) * g.B, U.len));
  if (max(lo, U.p0) >= hi) return false;
  U.rowi = row_index(U.r, U.kvh, U.i, g.Hkv, g.Nmax);
  U.lbase = list_row_base(U.r, U.kvh, U.i, g.Hkv, g.Nmax);
  int c = __ldg(a.cnt + U.rowi);
  if (c < 0 || c > U.i + 1) {
    atomicOr(g.status, FP_DEV_BAD_LIST);
    c = c < 0 ? 0 : U.i + 1;
  }
  U.count = c;
  return true;
}


// The producer's view of one visited key block: its index and, for a paged
// cache, the pool page of each page-sized sub-tile (at most BLK / 16 of them).
// Loaded one visit ahead (raw), checked when the visit's copies are issued.
template <int BLK>
struct TileSrc {
  int j;
  int page[BLK / 16];
};

__device__ __forceinline__ int checked_entry(const AttnArgs& a, const Unit& U, int j) {
  if (j < 0 || j > U.i) {
    atomicOr(a.g.status, FP_DEV_BAD_LIST);
    j = U.i;
  }
  return j;
}

// Raw page-table entries of the sub-tiles of block j (paged only).
template <int BLK>
__device__ __forceinline__ void load_pages(const AttnArgs& a, const Unit& U, TileSrc<BLK>& t) {
  const Geometry& g = a.g;
  const int sub_rows = g.page_size < BLK ? g.page_size : BLK;
  const int nsub = BLK / sub_rows;
  const int32_t* row = g.page_table + (long long)U.r * g.max_pages;
#pragma unroll
  for (int s = 0; s < BLK / 16; ++s) {
    const int tok = t.j * BLK + s * sub_rows;
    t.page[s] = (s < nsub && tok < U.len) ? __ldg(row + (tok >> g.page_shift)) : g.num_pages;
  }
}

// Copies of the K or V tile of a visited block whose pages were loaded raw:
// out-of-range page ids are reported and read as zeros (outside the pool).
template <bool FP8, int BLK, bool PAGED, int D>
__device__ __forceinline__ void issue_kv_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, const AttnArgs& a,
                                              const Unit& U, const TileSrc<BLK>& t) {
  using C = Cfg<FP8, BLK, D>;
  const Geometry& g = a.g;
  if constexpr (!PAGED) {
#pragma unroll
    for (int ch = 0; ch < C::DCH; ++ch)
      tma_load_3d(dst + ch * C::KV_CHUNK, map, bar, ch * C::CH_ELEMS, U.kvh, U.off + t.j * BLK);
  } else {
    const int sub_rows = g.page_size < BLK ? g.page_size : BLK;
    const int nsub = BLK / sub_rows;
#pragma unroll
    for (int s = 0; s < BLK / 16; ++s) {
      if (s >= nsub) break;
      const int tok = t.j * BLK + s * sub_rows;
      int page = t.page[s];
      if (tok < U.len && (page < 0 || page >= g.num_pages)) {
        atomicOr(g.status, FP_DEV_BAD_PAGE);
        page = g.num_pages;  // out of range -> the copy fills zeros
      }
      const int slot = tok & (g.page_size - 1);
#pragma unroll
      for (int ch = 0; ch < C::DCH; ++ch)
        tma_load_4d(dst + ch * C::KV_CHUNK + s * sub_rows * 128, map, bar, ch * C::CH_ELEMS, U.kvh, slot, page);
    }
  }
}

template <bool FP8, int BLK, bool PAGED, int D>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using C = Cfg<FP8, BLK, D>;
  constexpr int KS = C::K_STAGES, VS = C::V_STAGES, V8S = C::V8_STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + 2 * C::Q_TILE;
  uint8_t* sV = sK + KS * C::K_TILE;    // 16-bit V tiles (PV operand)
  uint8_t* sV8 = sV + VS * C::V_TILE;   // e4m3 V tiles as loaded (e4m3 inputs)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV8 + V8S * C::V8_TILE);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + KS;
  uint64_t* v_full = k_empty + KS;
  uint64_t* v_empty = v_full + VS;
  uint64_t* v8_full = v_empty + VS;   // [V8S]
  uint64_t* v8_empty = v8_full + V8S;  // [V8S]
  uint64_t* s_full = v8_empty + V8S;  // [2]
  uint64_t* p_full = s_full + 2;   // [M-tile][half of the keys]
  uint64_t* o_full = p_full + 4;   // [2]
  uint64_t* drain = o_full + 2;
  uint64_t* unit_full = drain + 1;             // [kUnitRing]
  uint64_t* unit_empty = unit_full + kUnitRing;  // [kUnitRing]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(unit_empty + kUnitRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* unit_ring = const_cast<int*>(reinterpret_cast<volatile int*>(abort_flag + 1));  // [kUnitRing]

  const Geometry& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(v_full + s, FP8 ? 64 : 1);  // e4m3: every converter thread arrives
      mbar_init(v_empty + s, 1);
    }
    for (int s = 0; s < V8S; ++s) {
      mbar_init(v8_full + s, 1);
      mbar_init(v8_empty + s, 64);
    }
    for (int m = 0; m < 2; ++m) {
      mbar_init(s_full + m, 1);
      mbar_init(p_full + 2 * m, 128);
      mbar_init(p_full + 2 * m + 1, 128);
      mbar_init(o_full + m, 1);
    }
    mbar_init(drain, 1);
    for (int k = 0; k < kUnitRing; ++k) {
      mbar_init(unit_full + k, 1);
      mbar_init(unit_empty + k, UnitConsumers<FP8>::value);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // Rows a.rows..127 of each M-tile are never written by the Q copies; keep them zero.
  if (a.rows < 128) {
    const int pad = (128 - a.rows) * 128;
    for (int x = threadIdx.x * 16; x < 2 * C::DCH * pad; x += kThreads * 16) {
      const int chunk = x / pad, o = x % pad;
      *reinterpret_cast<uint4*>(sQ + chunk * 128 * 128 + a.rows * 128 + o) = make_uint4(0, 0, 0, 0);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // With programmatic dependent launch the prologue above overlapped the
  // previous kernel (discovery); wait for its results before reading lists.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp >= 8) reg_dealloc<kControlRegs>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int kt = 0, vt = 0, qn = 0;  // ring positions (tiles a CTA moves stay far below 2^31)
      const uint32_t q_bytes = 2u * C::DCH * a.rows * 128u;
      constexpr int VLS = FP8 ? V8S : VS;
      constexpr int VL_TILE = FP8 ? C::V8_TILE : C::V_TILE;
      uint8_t* sVL = FP8 ? sV8 : sV;
      uint64_t* vl_full = FP8 ? v8_full : v_full;
      uint64_t* vl_empty = FP8 ? v8_empty : v_empty;
      bool ok = true;
      UnitIter it{a.queue, a.order, unit_ring, unit_full, unit_empty, abort_flag, g.status, true, false, a.num_units, 0, 0};
      for (long long u = it.step(true, ok); u < a.num_units && ok; u = it.step(false, ok)) {
        Unit U;
        if (!decode_unit(u, a, U) || U.count == 0) continue;
        ok = mbar_wait(q_empty, (uint32_t)(qn & 1) ^ 1u, abort_flag, g.status, FP_DEV_TIMEOUT);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, q_bytes);
        for (int mt = 0; mt < 2; ++mt) {
          const int t = U.off + U.i * g.B + (U.pair * 2 + mt) * a.Tm - U.p0;  // may precede the request:
                                                                               // those rows are never stored
#pragma unroll
          for (int ch = 0; ch < C::DCH; ++ch)
            tma_load_3d(sQ + mt * C::Q_TILE + ch * 128 * 128, &tmQ, q_full, ch * C::CH_ELEMS, U.kvh * g.G, t);
        }
        ++qn;
        // Tile sources run ahead of the copies: the list entry of visit n + 2
        // and the pages of visit n + 1 are loaded before the producer blocks on
        // the rings for visit n, so their latency hides behind those waits.
        const int32_t* lrow = a.idx + U.lbase;
        TileSrc<BLK> cur, nxt;
        cur.j = checked_entry(a, U, __ldg(lrow));
        if constexpr (PAGED) load_pages<BLK>(a, U, cur);
        int j_ahead = U.count > 1 ? __ldg(lrow + 1) : 0;
        for (int n = 0; n < U.count && ok; ++n) {
          if (n + 1 < U.count) {
            nxt.j = checked_entry(a, U, j_ahead);
            if constexpr (PAGED) load_pages<BLK>(a, U, nxt);
            if (n + 2 < U.count) j_ahead = __ldg(lrow + n + 2);
          }
          int st = (int)(kt % KS);
          ok = mbar_wait(k_empty + st, (uint32_t)((kt / KS) & 1) ^ 1u, abort_flag, g.status, FP_DEV_TIMEOUT);
          if (!ok) break;
          mbar_arrive_expect_tx(k_full + st, C::K_TILE);
          issue_kv_tile<FP8, BLK, PAGED, D>(sK + st * C::K_TILE, &tmK, k_full + st, a, U, cur);
          ++kt;
          // V: straight into the 16-bit ring (bf16) or into the e4m3 ring the converter reads
          st = (int)(vt % VLS);
          ok = mbar_wait(vl_empty + st, (uint32_t)((vt / VLS) & 1) ^ 1u, abort_flag, g.status, FP_DEV_TIMEOUT);
          if (!ok) break;
          mbar_arrive_expect_tx(vl_full + st, VL_TILE);
          issue_kv_tile<FP8, BLK, PAGED, D>(sVL + st * VL_TILE, &tmV, vl_full + st, a, U, cur);
          ++vt;
          cur = nxt;
        }
      }
      // Every copy this CTA issued lands before its shared memory is released,
      // also when another role gave up after this loop ended (on the normal
      // path the consumers have already seen these phases complete).
      for (int t = kt - 1; t >= 0 && t >= kt - KS; --t)
        mbar_drain(k_full + (int)(t % KS), (uint32_t)((t / KS) & 1), g.status, FP_DEV_TIMEOUT);
      for (int t = vt - 1; t >= 0 && t >= vt - VLS; --t)
        mbar_drain(vl_full + (int)(t % VLS), (uint32_t)((t / VLS) & 1), g.status, FP_DEV_TIMEOUT);
      if (qn > 0) mbar_drain(q_full, (uint32_t)((qn - 1) & 1), g.status, FP_DEV_TIMEOUT);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // QK: kind::f8f6f4 e4m3 (format 0) or kind::f16 bf16 (format 1);
      // PV: kind::f16, f16 (format 0) for e4m3 inputs or bf16 (format 1)
      const uint32_t fmt = FP8 ? 0u : 1u;
      const uint32_t idesc_qk = instr_desc(fmt, 128, BLK, 0, 0);
      const uint32_t idesc_pv = instr_desc(fmt, 128, D, 0, 1);  // N = head dim
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      int kt = 0, vt = 0, qn = 0;  // ring positions (tiles a CTA moves stay far below 2^31)
      int pn[2] = {0, 0};
      bool ok = true;

      // Descriptors of the tiles' first bytes; an operand at byte offset `off`
      // within the CTA's shared window is base + off / 16 (the start-address
      // field cannot carry: every address is below 256 KB).
      const uint64_t dQ = smem_desc_sw128(sQa, 16, 1024);
      const uint64_t dK = smem_desc_sw128(sKa, 16, 1024);
      const uint64_t dV = smem_desc_sw128(sVa, C::KV_CHUNK, 1024);
      auto issue_qk = [&](int mt, int kst) {
        const uint64_t a0 = dQ + (uint64_t)((mt * C::Q_TILE) >> 4);
        const uint64_t b0 = dK + (uint64_t)((kst * C::K_TILE) >> 4);
#pragma unroll
        for (int ks = 0; ks < C::QK_STEPS; ++ks) {
          const uint32_t boff = (uint32_t)(ks * 32);  // 32 bytes of K per MMA
          const uint32_t ch = boff / 128, in = boff % 128;
          const uint64_t ad = a0 + ((ch * 128 * 128 + in) >> 4);
          const uint64_t bd = b0 + ((ch * C::KV_CHUNK + in) >> 4);
          if (FP8) umma_f8_ss(tmem + mt * 128, ad, bd, idesc_qk, ks > 0);
          else umma_f16_ss(tmem + mt * 128, ad, bd, idesc_qk, ks > 0);
        }
      };
      // P occupies the first BLK / 2 columns of the M-tile's S region (16-bit pairs).
      auto issue_pv = [&](int mt, int vst, bool acc, int hf) {
        const uint64_t b0 = dV + (uint64_t)((vst * C::V_TILE) >> 4);
#pragma unroll
        for (int ks = hf * (C::PV_STEPS / 2); ks < (hf + 1) * (C::PV_STEPS / 2); ++ks) {
          const uint32_t a_t = tmem + mt * 128 + ks * (C::PV_KEYS / 2);
          const uint64_t bd = b0 + ((ks * C::PV_KEYS * 128) >> 4);
          umma_f16_ts(tmem + 256 + mt * 128, a_t, bd, idesc_pv, (acc || ks > 0) ? 1u : 0u);
        }
      };

      UnitIter it{a.queue, a.order, unit_ring, unit_full, unit_empty, abort_flag, g.status, false, false, a.num_units, 0, 0};
      for (long long u = it.step(true, ok); u < a.num_units && ok; u = it.step(false, ok)) {
        Unit U;
        if (!decode_unit(u, a, U) || U.count == 0) continue;
        ok = mbar_wait(q_full, (uint32_t)(qn & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
        if (!ok) break;
        ++qn;
        int kst = (int)(kt % KS);
        ok = mbar_wait(k_full + kst, (uint32_t)((kt / KS) & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
        if (!ok) break;
        tc_fence_after();
        issue_qk(0, kst);
        umma_commit(s_full + 0);
        issue_qk(1, kst);
        umma_commit(s_full + 1);
        umma_commit(k_empty + kst);
        ++kt;
        if (U.count == 1) umma_commit(q_empty);
        for (int n = 0; n < U.count; ++n) {
          const int vst = (int)(vt % VS);
          ok = mbar_wait(v_full + vst, (uint32_t)((vt / VS) & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
          if (!ok) break;
          ok = mbar_wait(p_full + 0, (uint32_t)(pn[0] & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
          if (!ok) break;
          tc_fence_after();
          issue_pv(0, vst, n > 0, 0);
          // the next K tile is waited for while softmax 0 finishes its second half,
          // so S0(n+1) follows PV0(n) without a gap
          const bool more = n + 1 < U.count;
          if (more) {
            kst = (int)(kt % KS);
            ok = mbar_wait(k_full + kst, (uint32_t)((kt / KS) & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
            if (!ok) break;
          }
          ok = mbar_wait(p_full + 1, (uint32_t)(pn[0] & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
          if (!ok) break;
          ++pn[0];
          tc_fence_after();
          issue_pv(0, vst, true, 1);
          if (more) {
            issue_qk(0, kst);
            umma_commit(s_full + 0);
          } else {
            umma_commit(o_full + 0);
          }
          ok = mbar_wait(p_full + 2, (uint32_t)(pn[1] & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
          if (!ok) break;
          tc_fence_after();
          issue_pv(1, vst, n > 0, 0);
          ok = mbar_wait(p_full + 3, (uint32_t)(pn[1] & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
          if (!ok) break;
          ++pn[1];
          tc_fence_after();
          issue_pv(1, vst, true, 1);
          umma_commit(v_empty + vst);
          ++vt;
          if (more) {
            issue_qk(1, kst);
            umma_commit(s_full + 1);
            umma_commit(k_empty + kst);
            ++kt;
            if (n + 2 == U.count) umma_commit(q_empty);
          } else {
            umma_commit(o_full + 1);
          }
        }
      }
      // every MMA this thread issued has completed once `drain` flips
      umma_commit(drain);
      mbar_drain(drain, 0u, g.status, FP_DEV_TIMEOUT);
    }
  } else if (FP8 && warp >= kConvertWarp) {
    // ------------------------------------------------------------------ V converter (e4m3 inputs)
    // Widens every V tile the producer loads, in the same order, from the e4m3
    // ring into the f16 ring the PV MMAs read; exact (e4m3 is a subset of f16).
    const int ct = threadIdx.x - kConvertWarp * 32;  // 0..63
    int vt = 0;
    bool ok = true;
    UnitIter it{a.queue, a.order, unit_ring, unit_full, unit_empty, abort_flag, g.status, false, true, a.num_units, 0, 0};
    for (long long u = it.step(true, ok); u < a.num_units && ok; u = it.step(false, ok)) {
      Unit U;
      if (!decode_unit(u, a, U) || U.count == 0) continue;
      for (int n = 0; n < U.count; ++n, ++vt) {
        constexpr int V8D = V8S > 0 ? V8S : 1;  // (this branch runs for e4m3 only)
        const int s8 = (int)(vt % V8D), s16 = (int)(vt % VS);
        ok = mbar_wait<true>(v8_full + s8, (uint32_t)((vt / V8D) & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
        if (!ok) break;
        ok = mbar_wait<true>(v_empty + s16, (uint32_t)((vt / VS) & 1) ^ 1u, abort_flag, g.status, FP_DEV_TIMEOUT);
        if (!ok) break;
        widen_v_tile<BLK>(sV8 + s8 * C::V8_TILE, sV + s16 * C::V_TILE, ct, 64);
        // the tensor cores read the tile through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(v_full + s16);
        mbar_arrive(v8_empty + s8);
      }
      if (!ok) break;
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax warpgroups
    reg_alloc<kSoftmaxRegs>();
    const int mt = warp >> 2;
    const int row = threadIdx.x - mt * 128;
    const uint32_t lane_base = (uint32_t)(row & ~31) << 16;
    const uint32_t tS = tmem + lane_base + mt * 128;
    const uint32_t tO = tmem + lane_base + 256 + mt * 128;
    const int hh = row % g.G, tt = row / g.G;
    int sn = 0, on = 0;
    bool ok = true;
    UnitIter it{a.queue, a.order, unit_ring, unit_full, unit_empty, abort_flag, g.status, false, true, a.num_units, 0, 0};
    for (long long u = it.step(true, ok); u < a.num_units && ok; u = it.step(false, ok)) {
      Unit U;
      if (!decode_unit(u, a, U)) continue;
      const int qtok = (U.pair * 2 + mt) * a.Tm + tt;  // token within the query block
      const int qpos = U.i * g.B + qtok;               // its position in the request
      const bool valid = row < a.rows && qpos >= U.p0 && qpos < U.len;
      const int h = U.kvh * g.G + hh;
      const long long orow = (long long)U.off + qpos - U.p0;
      float sl2 = a.scale_log2;
      float vmul = 1.f;
      if (FP8 && row < a.rows) {
        sl2 *= __ldg(g.q_scale + h) * __ldg(g.k_scale + U.kvh);
        vmul = __ldg(g.v_scale + U.kvh);
      }
      float m_ref = -INFINITY, l = 0.f;
      // Lists are strictly ascending, so only the last visit can be the
      // diagonal block (the producer validates every entry).
      const bool last_is_diag = U.count > 0 && __ldg(a.idx + U.lbase + U.count - 1) == U.i;
      // per-head selection: a visited block this row's head did not keep is masked
      const uint8_t* hbp = g.head_bits ? g.head_bits + U.lbase : nullptr;
      // (without head bits every head keeps every listed block, G up to 16)
      uint32_t hb_next = (hbp && U.count > 0) ? __ldg(hbp) : 0xFFFFFFFFu;
      for (int n = 0; n < U.count; ++n) {
        const uint32_t hb = hb_next;
        if (hbp && n + 1 < U.count) hb_next = __ldg(hbp + n + 1);  // one visit ahead
        ok = mbar_wait<true>(s_full + mt, (uint32_t)(sn & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
        if (!ok) break;
        ++sn;
        tc_fence_after();
        // S in two halves: the second half's TMEM load is in flight while the
        // first half is masked and reduced
        float s[BLK];
        const bool diag = last_is_diag && n == U.count - 1;  // keys after the query are masked
        const bool hmask = !((hb >> hh) & 1u);               // block not kept by this row's head
        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
        {
          uint32_t sr[BLK];
#pragma unroll
          for (int c = 0; c < BLK / 64; ++c) tmem_ld32(tS + c * 32, sr + c * 32);
          tmem_wait_ld();
#pragma unroll
          for (int c = BLK / 64; c < BLK / 32; ++c) tmem_ld32(tS + c * 32, sr + c * 32);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if (hf == 1) tmem_wait_ld();
#pragma unroll
            for (int c = hf * (BLK / 2); c < (hf + 1) * (BLK / 2); ++c) s[c] = __uint_as_float(sr[c]);
            if (diag || hmask) {
#pragma unroll
              for (int c = hf * (BLK / 2); c < (hf + 1) * (BLK / 2); ++c)
                if (hmask || c > qtok) s[c] = -INFINITY;
            }
#pragma unroll
            for (int c = hf * (BLK / 2); c < (hf + 1) * (BLK / 2); c += 8) {
              m0 = fmax3(m0, s[c], s[c + 1]);
              m1 = fmax3(m1, s[c + 2], s[c + 3]);
              m2 = fmax3(m2, s[c + 4], s[c + 5]);
              m3 = fmax3(m3, s[c + 6], s[c + 7]);
            }
          }
        }
        const float mx = fmax3(m0, m1, fmaxf(m2, m3));
        const float m_new = fmaxf(m_ref, mx * sl2);
        const bool need = m_new > m_ref + RescaleThreshold<FP8>::value;
        const float f = need ? fast_exp2(m_ref - (m_new - MaxOffset<FP8>::value)) : 1.f;
        if (need) {
          l *= f;
          m_ref = m_new - MaxOffset<FP8>::value;
        }
        // TMEM accesses are warp-collective: rescale when any row of the warp needs it
        if (n > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t r16[16];
            tmem_ld16(tO + c * 16, r16);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) r16[e] = __float_as_uint(__uint_as_float(r16[e]) * f);
            tmem_st16(tO + c * 16, r16);
          }
        }
        // P = 2^(s*sl2 - m_ref), computed where it is packed (bf16, or f16 for
        // e4m3 inputs). The row sum is taken over the rounded weights that the
        // PV MMA consumes, so O / l is an exact convex combination of V rows
        // and a dominant key's rounding cancels between numerator and denominator.
        float lsum0 = 0.f, lsum1 = 0.f, lsum2 = 0.f, lsum3 = 0.f;
        // (m_ref stays -inf while every visited block so far was masked for this row)
        const float negm = m_ref == -INFINITY ? 0.f : -m_ref;
        const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(negm, negm);
        // P goes out in two halves of the visited block's keys; the MMA issuer
        // starts O += P V on the first half while the second is computed.
        {
          constexpr int HALF = BLK / 2;              // keys per half
          constexpr int CH = HALF < 64 ? HALF : 64;  // keys per TMEM store
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
            for (int c = 0; c < HALF / CH; ++c) {
              const int k0 = hf * HALF + c * CH;
              uint32_t pk[CH / 2];
#pragma unroll
              for (int e = 0; e < CH / 2; ++e) {
                float p0, p1;
                exp2_pair(s[k0 + 2 * e], s[k0 + 2 * e + 1], sl2, m_ref, sl2x2, negm2, p0, p1);
                const uint32_t u = pack_p2<FP8>(p0, p1);
                pk[e] = u;
                if (e & 1) add_p2<FP8>(lsum2, lsum3, u);
                else add_p2<FP8>(lsum0, lsum1, u);
              }
              if constexpr (CH == 64) tmem_st32(tS + k0 / 2, pk);
              else tmem_st16(tS + k0 / 2, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full + 2 * mt + hf);
          }
        }
        l += (lsum0 + lsum1) + (lsum2 + lsum3);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16, natural-log LSE
      __nv_bfloat16* orow_ptr = a.o + (orow * g.Hq + h) * D;
      if (U.count == 0) {
        if (valid) {
          for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow_ptr)[c] = make_uint4(0, 0, 0, 0);
          if (a.lse) a.lse[(long long)h * a.T + orow] = -INFINITY;
        }
        continue;
      }
      ok = mbar_wait<true>(o_full + mt, (uint32_t)(on & 1), abort_flag, g.status, FP_DEV_TIMEOUT);
      if (!ok) break;
      ++on;
      tc_fence_after();
      const float inv = l > 0.f ? vmul / l : 0.f;  // a row that saw no key (masked everywhere) gets O = 0
      // the O row in TMEM round trips of 64 columns
#pragma unroll
      for (int hc = 0; hc < D / 64; ++hc) {
        uint32_t r[64];
        tmem_ld32(tO + hc * 64, r);
        tmem_ld32(tO + hc * 64 + 32, r + 32);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[8 * c + 2 * e]) * inv,
                                                              __uint_as_float(r[8 * c + 2 * e + 1]) * inv);
              pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            reinterpret_cast<uint4*>(orow_ptr + hc * 64)[c] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      if (valid && a.lse)
        a.lse[(long long)h * a.T + orow] = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
bool encode(CUtensorMap* m, bool fp8, int rank, const void* base, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  return encode_tiled(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims,
                      strides, box);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

template <bool FP8, int BLK, bool PAGED, int D>
fp_status_t run(const AttnArgs& a, const void* q, const void* k, const void* v, cudaStream_t s, bool pdl) {
  using C = Cfg<FP8, BLK, D>;
  const Geometry& g = a.g;
  const cuuint64_t es = FP8 ? 1 : 2;
  CUtensorMap mq, mk, mv;
  {
    const cuuint64_t dims[3] = {D, (cuuint64_t)g.Hq, (cuuint64_t)a.T};
    const cuuint64_t strides[2] = {D * es, (cuuint64_t)g.Hq * D * es};
    const cuuint32_t box[3] = {(cuuint32_t)C::CH_ELEMS, (cuuint32_t)g.G, (cuuint32_t)a.Tm};
    if (!encode(&mq, FP8, 3, q, dims, strides, box)) return FP_ERR_CUDA;
  }
  if (!PAGED) {
    const cuuint64_t dims[3] = {D, (cuuint64_t)g.Hkv, (cuuint64_t)a.T};
    const cuuint64_t strides[2] = {D * es, (cuuint64_t)g.Hkv * D * es};
    const cuuint32_t box[3] = {(cuuint32_t)C::CH_ELEMS, 1, (cuuint32_t)BLK};
    if (!encode(&mk, FP8, 3, k, dims, strides, box) || !encode(&mv, FP8, 3, v, dims, strides, box))
      return FP_ERR_CUDA;
  } else {
    const cuuint64_t P = (cuuint64_t)g.page_size;
    const cuuint64_t dims[4] = {D, (cuuint64_t)g.Hkv, P, (cuuint64_t)g.num_pages};
    const cuuint64_t strides[3] = {D * es, (cuuint64_t)g.Hkv * D * es, P * g.Hkv * D * es};
    const cuuint32_t box[4] = {(cuuint32_t)C::CH_ELEMS, 1, (cuuint32_t)(g.page_size < BLK ? g.page_size : BLK), 1};
    if (!encode(&mk, FP8, 4, k, dims, strides, box) || !encode(&mv, FP8, 4, v, dims, strides, box))
      return FP_ERR_CUDA;
  }
  auto kern = sparse_attention_kernel<FP8, BLK, PAGED, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) {
    set_last_error("attention smem attribute", (int)e, cudaGetErrorString(e));
    return FP_ERR_CUDA;
  }
  const long long grid = a.num_units < sm_count() ? a.num_units : sm_count();
  if (grid <= 0) return FP_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, a);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("attention launch", (int)e, cudaGetErrorString(e));
    return FP_ERR_CUDA;
  }
  return FP_OK;
}

}  // namespace

// Tokens per M-tile (Tm), M-tile pairs per query block and work units of the
// attention for this geometry; false when B / Tm is not an even number >= 2.
bool attention_layout(const Geometry& g, int& Tm, int& nPairs, long long& units) {
  Tm = 1;
  // at least two M-tiles per query block (a work unit is a pair of them): for
  // G = 1 at B = 128, or G <= 2 at B = 64, the M-tiles are half full
  while (Tm * 2 * g.G <= 128 && Tm * 2 <= g.B / 2) Tm *= 2;
  const int nM = g.B / Tm;
  if (nM < 2 || nM % 2 != 0) return false;
  nPairs = nM / 2;
  units = (long long)g.Nmax * g.R * g.Hkv * nPairs;
  return true;
}

long long attention_units(const Geometry& g) {
  int Tm, nPairs;
  long long units;
  return attention_layout(g, Tm, nPairs, units) ? units : 0;
}

namespace {

constexpr int kOrderThreads = 1024;

// Claim order for the device work queue, longest lists first: the work units
// sorted by their row's list length, descending (a counting sort over the
// lengths 0..Nmax; the M-tile pairs of one row stay together, rows of equal
// length in arbitrary order). One CTA; it also zeroes the queue counter.
__global__ void __launch_bounds__(kOrderThreads)
    unit_order_kernel(const Geometry g, int nPairs, const int32_t* __restrict__ cnt, int* __restrict__ order,
                      int* __restrict__ queue) {
  // the attention, launched as a programmatic dependent, may start its prologue
  asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ int start[];  // [Nmax + 1]: rows per length, then first unit position per length
  __shared__ int warp_tot[kOrderThreads / 32];
  const int bins = g.Nmax + 1;
  const long long rows = (long long)g.R * g.Hkv * g.Nmax;
  auto key = [&](long long row) {
    const int c = __ldg(cnt + row);
    return c < 0 ? 0 : (c > g.Nmax ? g.Nmax : c);
  };
  for (int b = threadIdx.x; b < bins; b += kOrderThreads) start[b] = 0;
  if (threadIdx.x == 0) *queue = 0;
  __syncthreads();
  for (long long row = threadIdx.x; row < rows; row += kOrderThreads) atomicAdd(&start[key(row)], 1);
  __syncthreads();
  // exclusive prefix over the lengths in descending order (thread t owns a run of them)
  const int per = (bins + kOrderThreads - 1) / kOrderThreads;
  const int d0 = threadIdx.x * per, d1 = min(d0 + per, bins);
  int local = 0;
  for (int d = d0; d < d1; ++d) local += start[bins - 1 - d];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += warp_tot[w];
  int run = before + incl - local;  // rows of longer lists
  for (int d = d0; d < d1; ++d) {
    const int b = bins - 1 - d, n = start[b];
    start[b] = run * nPairs;
    run += n;
  }
  __syncthreads();
  const int RH = g.R * g.Hkv;
  for (long long row = threadIdx.x; row < rows; row += kOrderThreads) {
    const int pos = atomicAdd(&start[key(row)], nPairs);
    const int i = (int)(row % g.Nmax), rk = (int)(row / g.Nmax);  // rk = r * Hkv + kvh
    const int u0 = ((g.Nmax - 1 - i) * RH + rk) * nPairs;
    for (int p = 0; p < nPairs; ++p) order[pos + p] = u0 + p;
  }
}

}  // namespace

cudaError_t launch_unit_order(const Geometry& g, const int32_t* cnt, int* order, int* queue, cudaStream_t s) {
  int Tm, nPairs;
  long long units;
  if (!attention_layout(g, Tm, nPairs, units)) return cudaErrorInvalidValue;
  unit_order_kernel<<<1, kOrderThreads, (size_t)(g.Nmax + 1) * sizeof(int), s>>>(g, nPairs, cnt, order, queue);
  return cudaGetLastError();
}

fp_status_t launch_attention(const Geometry& g, const void* q, const void* k, const void* v, const int32_t* idx,
                             const int32_t* cnt, void* o, float* lse, cudaStream_t s, int* queue, const int* order,
                             bool pdl) {
  AttnArgs a;
  a.queue = queue;
  a.order = order;
  a.g = g;
  int Tm, nPairs;
  long long units;
  if (!attention_layout(g, Tm, nPairs, units)) return FP_ERR_UNSUPPORTED;
  if (units >= INT_MAX) return FP_ERR_UNSUPPORTED;  // int unit ids
  a.Tm = Tm;
  a.rows = Tm * g.G;
  a.nPairs = nPairs;
  a.num_units = units;
  a.T = g.cu ? (long long)g.total_tokens : (long long)g.R * g.L;
  a.scale_log2 = g.scale * 1.4426950408889634f;
  a.idx = idx;
  a.cnt = cnt;
  a.o = reinterpret_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  const bool paged = g.page_table != nullptr;
  if (g.d == 128) {
    if (g.B == 128) {
      if (g.fp8) return paged ? run<true, 128, true, 128>(a, q, k, v, s, pdl) : run<true, 128, false, 128>(a, q, k, v, s, pdl);
      return paged ? run<false, 128, true, 128>(a, q, k, v, s, pdl) : run<false, 128, false, 128>(a, q, k, v, s, pdl);
    }
    if (g.B == 64) {
      if (g.fp8) return paged ? run<true, 64, true, 128>(a, q, k, v, s, pdl) : run<true, 64, false, 128>(a, q, k, v, s, pdl);
      return paged ? run<false, 64, true, 128>(a, q, k, v, s, pdl) : run<false, 64, false, 128>(a, q, k, v, s, pdl);
    }
  }
  if (g.d == 64 && !g.fp8) {  // e4m3 rows of 64 bytes are not supported
    if (g.B == 128)
      return paged ? run<false, 128, true, 64>(a, q, k, v, s, pdl) : run<false, 128, false, 64>(a, q, k, v, s, pdl);
    if (g.B == 64)
      return paged ? run<false, 64, true, 64>(a, q, k, v, s, pdl) : run<false, 64, false, 64>(a, q, k, v, s, pdl);
  }
  return FP_ERR_UNSUPPORTED;
}

}  // namespace fp
