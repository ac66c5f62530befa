// prefill.cu -- fused causal prefill attention over precision-grouped tile
// traversals (TriAttention abstract: one fused kernel skips omitted tiles and
// merges both QK precisions into a single normalised output; TileMix abstract:
// each tile group goes through a high-precision or an INT8 score path and both
// paths update the same online-softmax state).
//
// Work unit: one query head h of one sequence b and one pair of q-tiles
// (2j, 2j+1) = 128 query rows, the M of one tcgen05 MMA (rows 0-63 q-tile 2j =
// TMEM lanes 0-63, rows 64-127 q-tile 2j+1 = lanes 64-127).  The two q-tiles'
// CSR traversals (each sorted by (precision, kt): three ascending runs) are
// merged into one stream of key tiles in ascending kt; an entry carries the
// precision each q-tile gives the tile (or none).  When the two precisions
// differ, the entry computes both score products into the same S block, each
// MMA writing only its own q-tile's 64 lanes (tcgen05.mma output-lane mask), so
// every entry has one S block, one softmax pass over all 128 rows and one P V.
//
// Two work units share one CTA (384 threads) so that one unit's softmax runs
// while the tensor core works on the other's tiles:
//   warps 0, 2  TMA producers of units 0, 1: the unit's Q operands once (INT8
//               codes; INT4 codes in their int8 operand form, 16 x code, as the
//               quantiser writes them; BF16), then per entry one K tile per
//               precision the entry needs into the unit's K ring and the BF16 V
//               tile into its V ring;
//   warps 1, 3  MMA issuers of units 0, 1 (warp 1 also owns TMEM): S = Q K^T with
//               kind::i8 (INT8 / INT4, exact int32) or kind::f16 (BF16, fp32) into
//               one of the unit's two S blocks in TMEM, then O += P V with P read
//               from TMEM (bf16, written over S) and V from shared memory;
//   warps 4-7   softmax / epilogue of unit 0, warps 8-11 of unit 1: one thread
//               per query row (TMEM lane): S -> log2-domain scores -> mask ->
//               online softmax with lazy rescaling of O -> bf16 P into TMEM;
//               finally O / l.  With two S blocks, QK(i+1) runs while entry i is
//               in the softmax.
// The producer and MMA warps run converged, every lane computing the same
// (warp-uniform) operands; elect.sync picks the one lane that issues each TMA
// copy, MMA, commit and arrive, and waits are left by the warp as a whole.
// Every ring belongs to one unit: one filler and one consumer, both taking its
// slots in order, so no parity wait can alias a phase two uses away.  All waits
// are bounded (2 s); on expiry a role records TRA_DEV_TIMEOUT and all drain.
#include <type_traits>

#include "tra_device.cuh"
#include "tra_launch.h"

namespace tra {
namespace {

constexpr int kThreads = 384;
constexpr int kUnits = 2;
// log2 units: O and l are rescaled only once the running max has grown by more
// than 2^16.  Until then P (bf16, exponent range of fp32) may reach 2^16, and
// with fewer than 2^31 keys per row l < 2^47 and |O| < 2^47 * max|V| stay far
// inside fp32; rarer rescales matter because each one waits for the previous
// P V to complete.
constexpr float kRescaleThreshold = 16.0f;
constexpr int kSmemLimit = 232448;  // max dynamic shared memory per CTA on sm_100
constexpr uint32_t kNoKt = 0x0FFFFFFFu;

// Precision of a hybrid-prefill entry whose K and V come from the mixed operands
// (bf16 rows of selected tokens, INT4 codes as bf16 integers for the others).
constexpr int kPrecHyb = 5;

template <int D, int MODE>
struct Cfg {
  static constexpr bool kHyb = MODE == kPrefillModeHybrid;        // token-level hybrid prefill
  static constexpr bool kHasF8 = MODE == kPrefillModeBoundaryF8;   // FP8 band of a boundary policy
  static constexpr bool kHasBf16 = MODE != TRA_POLICY_BOUNDARY && !kHasF8;  // bf16 Q and K operands
  static constexpr bool kHasInt4 = MODE != TRA_POLICY_BITMASK && !kHyb;  // INT4 operands (int8 form)
  static constexpr int kMode = MODE;
  // fp32 score tiles (BF16, FP8, hybrid) occur beside the integer ones
  static constexpr bool kFloatScores = kHasBf16 || kHasF8;
  // work units per CTA: two, or one under a mixed policy, whose operand buffers
  // (int8, INT4 and bf16 Q, bf16-sized K slots) do not fit twice
  static constexpr int kCtaUnits = MODE == TRA_POLICY_MIXED ? 1 : 2;
  static constexpr int kQ8Bytes = kHyb ? 0 : 128 * D;          // int8 Q codes
  static constexpr int kQ4Bytes = kHasInt4 ? 128 * D : 0;      // INT4 Q codes as int8
  static constexpr int kQbBytes = kHasBf16 ? 128 * D * 2 : 0;  // bf16 Q
  static constexpr int kQfBytes = kHasF8 ? 128 * D : 0;        // FP8 E4M3 Q codes
  static constexpr int kQUnitBytes = kQ8Bytes + kQ4Bytes + kQbBytes + kQfBytes;
  // K slot: one K tile, BF16 or int8 codes (INT8 or INT4 in int8 form)
  static constexpr int kKBytes = kHasBf16 ? 64 * D * 2 : 64 * D;
  static constexpr int kVBytes = 64 * D * 2;
  static constexpr int kBase = kCtaUnits * kQUnitBytes + 2048 + 1024;  // + barriers, slack
  // ring depths per unit: as many of both as fit, K first (up to 4 each)
  static constexpr int kRoom = (kSmemLimit - kBase) / kCtaUnits;
  static constexpr int kStagesK = kRoom >= 4 * kKBytes + 4 * kVBytes ? 4
                                  : kRoom >= 3 * kKBytes + 3 * kVBytes ? 3 : 2;
  static constexpr int kStagesVFit = (kRoom - kStagesK * kKBytes) / kVBytes;
  static constexpr int kStagesV = kStagesVFit > 4 ? 4 : kStagesVFit;
  static_assert(kStagesV >= 2, "shared memory too small for the V rings");
  static constexpr int kOffQ = 0;                                             // unit u at u * kQUnitBytes
  static constexpr int kOffK = kCtaUnits * kQUnitBytes;                       // [unit][slot]
  static constexpr int kOffV = kOffK + kCtaUnits * kStagesK * kKBytes;
  static constexpr int kOffBar = kOffV + kCtaUnits * kStagesV * kVBytes;
  // (barriers exist for two units in every mode; a CTA's missing second unit has
  // no entries and touches none of the buffers above)
  static constexpr int kUnitBars = 2 * kStagesK + 2 * kStagesV + 6;
  static constexpr int kNumBars = 1 + kUnits * kUnitBars + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= kSmemLimit, "shared memory budget");
  // int8 K-major rows of D bytes: 128-byte swizzle for D = 128, 64-byte for D = 64
  static constexpr uint32_t kI8Layout = D == 128 ? kSwz128 : kSwz64;
  static constexpr uint32_t kI8Sbo = D == 128 ? 1024 : 512;
  static constexpr int kSlabs = D / 64;  // bf16 64-element (128-byte) slabs per row
  // TMEM columns of unit u: S/P buffer b at u*256 + 64*b (P, bf16 pairs, in its
  // first 32 columns), O at u*256+128
  static constexpr uint32_t kTmemCols = 512;
};

// The two q-tiles' rows of a unit merged in ascending kt.  A row lists its tiles
// as ascending runs, one per precision, in increasing precision code (entries are
// sorted as whole words); PR are the precisions a mode's lists can hold, so the
// merge walks only those runs.  next() yields each kt of either row once with the
// precision each row gives it (0: the row does not list it).
template <int... PR>
struct KtMerge {
  static constexpr int NR = sizeof...(PR);
  __host__ __device__ static constexpr int prec(int g) {
    constexpr int a[NR] = {PR...};
    return a[g];
  }
  const uint32_t* e;
  int pos[2][NR], end[2][NR];
  uint32_t head[2][NR];  // current kt of each run, kNoKt when exhausted

  __device__ __forceinline__ void load(int r, int g) {
    head[r][g] = pos[r][g] < end[r][g] ? (__ldg(e + pos[r][g]) & kNoKt) : kNoKt;
  }
  __device__ __forceinline__ static int lower_bound(const uint32_t* e, int lo, int hi, uint32_t key) {
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(e + mid) < key) lo = mid + 1; else hi = mid;
    }
    return lo;
  }
  // rows [rs[r], re[r]) of the entry array; an absent row is empty.  len[r][g]: the
  // length of run g when the policy fixes it (boundary rows), or -1 to find the run's
  // end by binary search; a length is clamped to the row.
  __device__ __forceinline__ void init(const uint32_t* entries, const int (&rs)[2], const int (&re)[2],
                                       const int (&len)[2][NR]) {
    e = entries;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      int lo = rs[r];
#pragma unroll
      for (int g = 0; g < NR; ++g) {  // run g holds precision prec(g)
        int hi = re[r];
        if (g + 1 < NR)
          hi = len[r][g] >= 0 ? min(lo + len[r][g], re[r])
                              : lower_bound(e, lo, re[r], (uint32_t)prec(g + 1) << 28);
        pos[r][g] = lo;
        end[r][g] = hi;
        lo = hi;
      }
#pragma unroll
      for (int g = 0; g < NR; ++g) load(r, g);
    }
  }
  // next entry: kt and each row's precision (TRA_PREC_*, or 0)
  __device__ __forceinline__ bool next(int& kt, int& p0, int& p1) {
    uint32_t k = kNoKt;
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int g = 0; g < NR; ++g) k = min(k, head[r][g]);
    if (k == kNoKt) return false;
    int pr[2] = {0, 0};
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int g = 0; g < NR; ++g)
        if (head[r][g] == k) {
          pr[r] = prec(g);
          ++pos[r][g];
          load(r, g);
        }
    kt = (int)k;
    p0 = pr[0];
    p1 = pr[1];
    return true;
  }
};

// One work unit: query head h of sequence b, q-tiles (2j, 2j+1).
struct Unit {
  bool valid, has_second;
  int h, b, kvh, qt0, nt, T, seq0, toff, row0;
};

// Unit `id` in launch order: heaviest q-tile pairs (largest j) first, heads fastest.
__device__ __forceinline__ Unit make_unit(const PrefillParams& p, long long id) {
  Unit x;
  const long long total = (long long)p.jmax * p.B * p.Hq;
  x.h = (int)(id % p.Hq);
  x.b = (int)((id / p.Hq) % p.B);
  x.kvh = x.h / (p.Hq / p.Hkv);
  x.qt0 = 2 * (p.jmax - 1 - (int)(id / ((long long)p.Hq * p.B)));
  x.valid = false;
  x.seq0 = x.T = x.nt = x.toff = x.row0 = 0;
  x.has_second = false;
  if (id < total) {
    x.seq0 = __ldg(p.cu + x.b);
    x.T = __ldg(p.cu + x.b + 1) - x.seq0;
    x.nt = (x.T + kTile - 1) / kTile;
    x.valid = x.qt0 < x.nt;
  }
  if (x.valid) {
    x.toff = seq_tile_offset(p.cu, x.b);
    x.has_second = x.qt0 + 1 < x.nt;
    x.row0 = x.h * p.ntiles + x.toff + x.qt0;
  }
  return x;
}

// The last key tile a unit's causal rows can list (its second q-tile's diagonal).
// A list entry beyond it is reported as a bad list: no copy is issued for it and
// no per-tile array is indexed with it.
__device__ __forceinline__ int unit_kt_max(const Unit& x) { return x.qt0 + (x.has_second ? 1 : 0); }

// the precisions each prefill mode's traversal rows can hold
template <int MODE> struct MergeOf { using T = KtMerge<TRA_PREC_INT4, TRA_PREC_INT8>; };
template <> struct MergeOf<TRA_POLICY_BITMASK> { using T = KtMerge<TRA_PREC_INT8, TRA_PREC_BF16>; };
template <> struct MergeOf<TRA_POLICY_MIXED> {
  using T = KtMerge<TRA_PREC_INT4, TRA_PREC_INT8, TRA_PREC_BF16>;
};
template <> struct MergeOf<kPrefillModeBoundaryF8> {
  using T = KtMerge<TRA_PREC_INT4, TRA_PREC_INT8, TRA_PREC_FP8>;
};

template <class M, bool kClosedForm>
__device__ __forceinline__ M unit_merge(const PrefillParams& p, const Unit& x) {
  M c;
  int rs[2] = {0, 0}, re[2] = {0, 0};
  if (x.valid) {
    rs[0] = __ldg(p.row_ptr + x.row0);
    re[0] = rs[1] = __ldg(p.row_ptr + x.row0 + 1);
    re[1] = x.has_second ? __ldg(p.row_ptr + x.row0 + 2) : rs[1];
  }
  int len[2][M::NR];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int g = 0; g < M::NR; ++g) len[r][g] = -1;
  if constexpr (kClosedForm) {
    // boundary rows in closed form: the row keeps n = min(qt + 1, b2) tiles, the
    // nearest min(qt + 1, b1) INT8, then min(qt + 1, b8) - that FP8, the rest INT4,
    // written as the INT4 run, the INT8 run, the FP8 run
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int qt = x.qt0 + r;
      const int n8 = min(qt + 1, p.b1[x.h]);
      const int nf = min(qt + 1, p.b8[x.h]) - n8;
      len[r][0] = max(0, re[r] - rs[r] - n8 - nf);  // INT4
      if (M::NR > 2) len[r][1] = n8;                 // INT8 (before FP8)
    }
  }
  c.init(p.entries, rs, re, len);
  return c;
}

// The hybrid prefill's stream for one unit (q-tiles qt0, qt0 + 1): first every key
// tile that holds, for some row of the unit, keys outside the row's window (kPrecHyb:
// the mixed operands), then every tile that holds keys inside it (BF16: the original
// K and V).  A tile on a window's edge appears in both, each entry keeping only its
// own keys (the softmax masks by position).  Per q-tile qt: keys outside the window
// lie in tiles kt <= hhi(qt) = floor((64 qt + 63 - window) / 64), keys inside it in
// tiles wlo(qt) <= kt <= qt with wlo(qt) = max(0, floor((64 qt - window + 1) / 64)).
struct HybStream {
  int kt, hhi0, hhi1, wlo0, wlo1, qt0;
  bool second, in_window, any_window;
  __device__ __forceinline__ void init(const Unit& x, int window) {
    qt0 = x.qt0;
    second = x.valid && x.has_second;
    any_window = x.valid && window > 0;
    hhi0 = x.valid ? (64 * qt0 + 63 - window) >> 6 : -1;  // arithmetic shift: floor
    hhi1 = second ? (64 * (qt0 + 1) + 63 - window) >> 6 : -1;
    wlo0 = max(0, (64 * qt0 - window + 1) >> 6);
    wlo1 = max(0, (64 * (qt0 + 1) - window + 1) >> 6);
    kt = 0;
    in_window = false;
  }
  __device__ __forceinline__ bool next(int& kt_, int& p0, int& p1) {
    while (true) {
      if (!in_window) {
        if (kt <= max(hhi0, hhi1)) {
          p0 = kt <= hhi0 ? kPrecHyb : 0;
          p1 = kt <= hhi1 ? kPrecHyb : 0;
          kt_ = kt++;
          return true;
        }
        if (!any_window) return false;
        in_window = true;
        kt = second ? min(wlo0, wlo1) : wlo0;
      }
      const int kmax = second ? qt0 + 1 : qt0;
      if (kt > kmax) return false;
      p0 = (kt >= wlo0 && kt <= qt0) ? TRA_PREC_BF16 : 0;
      p1 = (second && kt >= wlo1) ? TRA_PREC_BF16 : 0;
      kt_ = kt++;
      if (p0 | p1) return true;
    }
  }
};

// the entry stream of a unit: the merged traversal rows, or the hybrid's own
template <class C>
__device__ __forceinline__ auto unit_stream(const PrefillParams& p, const Unit& x) {
  if constexpr (C::kHyb) {
    HybStream c;
    c.init(x, p.window);
    return c;
  } else {
    return unit_merge<typename MergeOf<C::kMode>::T,
                      C::kMode == TRA_POLICY_BOUNDARY || C::kMode == kPrefillModeBoundaryF8>(p, x);
  }
}

// The K tiles of an entry: one per distinct precision, q-tile 2j's first.
__device__ __forceinline__ int entry_fills(int p0, int p1) { return (p0 && p1 && p0 != p1) ? 2 : 1; }
__device__ __forceinline__ int entry_fill_prec(int p0, int p1, int f) {
  return f == 0 ? (p0 ? p0 : p1) : p1;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// tcgen05.mma with an output-lane mask: lanes whose bit is set in m0..m3 (lane
// 32 w + i <-> bit i of m_w) keep their contents.  Issued by one elected lane of a
// converged warp (all lanes pass the same operands).
__device__ __forceinline__ void mma_i8_mask(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                            uint32_t accumulate, const uint32_t (&m)[4]) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(m[0]), "r"(m[1]), "r"(m[2]), "r"(m[3])
      : "memory");
}
__device__ __forceinline__ void mma_bf16_mask(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                              uint32_t accumulate, const uint32_t (&m)[4]) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(m[0]), "r"(m[1]), "r"(m[2]), "r"(m[3])
      : "memory");
}

__device__ __forceinline__ void mma_f8_mask(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                            uint32_t accumulate, const uint32_t (&m)[4]) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(m[0]), "r"(m[1]), "r"(m[2]), "r"(m[3])
      : "memory");
}

// O += P V with the 128 x 16 bf16 A operand (P) read from TMEM (elected lane).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ PrefillMaps m) {
  using C = Cfg<D, MODE>;
  constexpr int NSK = C::kStagesK, NSV = C::kStagesV;
  extern __shared__ uint8_t smem_raw[];

  // ---- the CTA's work units (the second is absent under a mixed policy)
  auto unit_of = [&](int u) {
    const long long none = (long long)p.jmax * p.B * p.Hq;  // an id past the last unit
    return make_unit(p, u < C::kCtaUnits ? (long long)blockIdx.x * C::kCtaUnits + u : none);
  };
  const Unit un0 = unit_of(0);
  const Unit un1 = unit_of(1);
  if (!un0.valid && !un1.valid) return;  // uniform exit, before any barrier or TMEM use
  // INT4 operands exist only for policies with an INT4 region; a list entry asking
  // for INT4 without them is reported, never read
  const bool int4 = C::kHasInt4 && p.has_int4;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - smem_u32(smem_raw));
  auto sQ8 = [&](int u) { return base + C::kOffQ + u * C::kQUnitBytes; };
  auto sQ4 = [&](int u) { return base + C::kOffQ + u * C::kQUnitBytes + C::kQ8Bytes; };
  auto sQb = [&](int u) { return base + C::kOffQ + u * C::kQUnitBytes + C::kQ8Bytes + C::kQ4Bytes; };
  auto sQf = [&](int u) {
    return base + C::kOffQ + u * C::kQUnitBytes + C::kQ8Bytes + C::kQ4Bytes + C::kQbBytes;
  };
  auto sK = [&](int u, int s) { return base + C::kOffK + (u * NSK + s) * C::kKBytes; };
  auto sV = [&](int u, int s) { return base + C::kOffV + (u * NSV + s) * C::kVBytes; };
  const uint32_t bars = base + C::kOffBar;
  const uint32_t bar_q = bars;
  // barriers of unit u: K ring full/free, V ring full/free, then S full (2),
  // P full (2), O full, O final
  auto ubar = [&](int u, int k) { return bars + (1 + u * C::kUnitBars + k) * 8; };
  auto bar_kfull = [&](int u, int s) { return ubar(u, s); };
  auto bar_kfree = [&](int u, int s) { return ubar(u, NSK + s); };
  auto bar_vfull = [&](int u, int s) { return ubar(u, 2 * NSK + s); };
  auto bar_vfree = [&](int u, int s) { return ubar(u, 2 * NSK + NSV + s); };
  constexpr int kSB = 2 * NSK + 2 * NSV;  // first S/P/O barrier of a unit
  auto bar_sfull = [&](int u, int sb) { return ubar(u, kSB + sb); };
  auto bar_pfull = [&](int u, int sb) { return ubar(u, kSB + 2 + sb); };
  auto bar_ofull = [&](int u) { return ubar(u, kSB + 4); };
  // completes once every MMA of unit u (its last P V included) is done
  auto bar_ofinal = [&](int u) { return ubar(u, kSB + 5); };
  const uint32_t bar_done = bars + (1 + kUnits * C::kUnitBars) * 8;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::kOffMisc);
  volatile int* const err = reinterpret_cast<volatile int*>(gbase + C::kOffMisc + 16);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, kUnits);  // one arrival (with its byte count) per producer
    for (int u = 0; u < kUnits; ++u) {
      for (int s = 0; s < NSK; ++s) {
        mbar_init(bar_kfull(u, s), 1);
        mbar_init(bar_kfree(u, s), 1);
      }
      for (int s = 0; s < NSV; ++s) {
        mbar_init(bar_vfull(u, s), 1);
        mbar_init(bar_vfree(u, s), 1);
      }
      for (int sb = 0; sb < 2; ++sb) {
        mbar_init(bar_sfull(u, sb), 1);
        mbar_init(bar_pfull(u, sb), 128);
      }
      mbar_init(bar_ofull(u), 1);
      mbar_init(bar_ofinal(u), 1);
    }
    mbar_init(bar_done, kUnits);  // one commit per MMA-issuing thread
    *err = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // a wait left by the whole (converged) warp together: true when every lane saw
  // the phase complete
  auto wwait = [&](uint32_t bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, err));
  };

  if (warp == 0 || warp == 2) {
    // ================================================================ TMA producers
    // one warp per unit, each walking its own unit's merged stream into its own
    // rings.  The whole warp runs it with warp-uniform values; one elected lane
    // issues each copy and arrive, and a wait is left by all lanes together.
    {
      const int u = warp >> 1;
      const Unit x = u ? un1 : un0;
      const uint32_t qbytes =
          x.valid ? C::kQ8Bytes + (int4 ? C::kQ4Bytes : 0) + C::kQbBytes + C::kQfBytes : 0u;
      mbar_arrive_expect_tx_e(bar_q, qbytes);
      if (x.valid) {
        if (!C::kHyb) tma_load_2d_e(sQ8(u), &m.q8, bar_q, 0, x.row0 * kTile);
        if (int4) tma_load_2d_e(sQ4(u), &m.q4x, bar_q, 0, x.row0 * kTile);
        if (C::kHasF8) tma_load_2d_e(sQf(u), &m.qf8, bar_q, 0, x.row0 * kTile);
        if (C::kHasBf16) {
          for (int sl = 0; sl < C::kSlabs; ++sl)
            tma_load_3d_e(sQb(u) + sl * 128 * 128, &m.qb, bar_q, sl * 64, x.h,
                          x.seq0 + x.qt0 * kTile);
        }
      }
      auto c = unit_stream<C>(p, x);
      int kt, p0, p1;
      int nk = 0, nv = 0;  // fills issued so far into this unit's K and V rings
      while (c.next(kt, p0, p1)) {
        if (((p0 == TRA_PREC_INT4 || p1 == TRA_PREC_INT4) && !int4) ||
            (!C::kHasF8 && (p0 == TRA_PREC_FP8 || p1 == TRA_PREC_FP8)) || kt > unit_kt_max(x)) {
          *err = TRA_DEV_BAD_LIST;
          break;
        }
        bool ok = true;
        const int nf = entry_fills(p0, p1);
        for (int f = 0; f < nf; ++f) {
          const int prec = entry_fill_prec(p0, p1, f);
          const int s = nk % NSK, use = nk / NSK;  // the unit's K ring slot
          if (use > 0 && !wwait(bar_kfree(u, s), (use - 1) & 1)) { ok = false; break; }
          const uint32_t dst = sK(u, s);
          const int krow = (x.kvh * p.ntiles + x.toff + kt) * kTile;
          if (C::kHasBf16 && (prec == TRA_PREC_BF16 || prec == kPrecHyb)) {
            const CUtensorMap* km = prec == kPrecHyb ? &m.kmix : &m.kb;
            mbar_arrive_expect_tx_e(bar_kfull(u, s), 64 * D * 2);
            for (int sl = 0; sl < C::kSlabs; ++sl)
              tma_load_3d_e(dst + sl * 64 * 128, km, bar_kfull(u, s), sl * 64, x.kvh,
                            x.seq0 + kt * kTile);
          } else {
            mbar_arrive_expect_tx_e(bar_kfull(u, s), 64 * D);
            tma_load_2d_e(dst, prec == TRA_PREC_INT8 ? &m.k8 : prec == TRA_PREC_FP8 ? &m.kf8 : &m.k4x,
                          bar_kfull(u, s), 0, krow);
          }
          ++nk;
        }
        if (!ok) break;
        const int sv = nv % NSV, usev = nv / NSV;  // the unit's V ring slot
        if (usev > 0 && !wwait(bar_vfree(u, sv), (usev - 1) & 1)) break;
        // V of the entry: the mixed operand for a hybrid entry, else bf16 V
        const CUtensorMap* vm = (p0 == kPrecHyb || p1 == kPrecHyb) ? &m.vmix : &m.vb;
        mbar_arrive_expect_tx_e(bar_vfull(u, sv), 64 * D * 2);
        for (int sl = 0; sl < C::kSlabs; ++sl)
          tma_load_3d_e(sV(u, sv) + sl * 64 * 128, vm, bar_vfull(u, sv), sl * 64, x.kvh,
                        x.seq0 + kt * kTile);
        ++nv;
      }
      if (*err) {
        // an abandoned traversal: every load this warp issued lands before the CTA
        // can exit. Only this warp arrives on a full barrier, so the last fill of
        // each slot completes its phase as soon as its bytes are in.
        mbar_wait_drain(bar_q, 0);
        for (int s = 0; s < NSK && s < nk; ++s)
          mbar_wait_drain(bar_kfull(u, s), (uint32_t)(((nk - 1 - s) / NSK) & 1));
        for (int s = 0; s < NSV && s < nv; ++s)
          mbar_wait_drain(bar_vfull(u, s), (uint32_t)(((nv - 1 - s) / NSV) & 1));
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ================================================================ MMA issuers
    // The whole warp runs the issuer with warp-uniform values; one elected lane
    // issues each MMA and commit.
    {
      const int mu = warp >> 1;  // the unit this warp issues for
      constexpr uint32_t kIdI8 = instr_desc(2, 1, 0, 0, 64, 128);
      constexpr uint32_t kIdQK16 = instr_desc(1, 1, 0, 0, 64, 128);
      constexpr uint32_t kIdF8 = instr_desc(1, 0, 0, 0, 64, 128);  // f32 <- E4M3 x E4M3
      constexpr uint32_t kIdPV = instr_desc(1, 1, 0, 1, D, 128);
      const uint32_t tU = tmem + mu * 256;
      // Operand descriptors, built once: a K step (or a block of V rows) moves only
      // the start address, the descriptor's low bits in 16-byte units
      const uint64_t dQ8 = smem_desc(sQ8(mu), 16, C::kI8Sbo, C::kI8Layout);
      const uint64_t dQ4 = smem_desc(sQ4(mu), 16, C::kI8Sbo, C::kI8Layout);
      const uint64_t dQf = smem_desc(sQf(mu), 16, C::kI8Sbo, C::kI8Layout);
      const uint64_t dQb = smem_desc(sQb(mu), 16, 1024, kSwz128);
      bool ok = wwait(bar_q, 0);
      tc_fence_after();
      // O += P(idx) V(idx): P from TMEM buffer idx & 1, V (MN-major) from the unit's
      // V ring, which holds one tile per entry of the unit, in order
      // hi_lo: a mixed-operand entry of the hybrid prefill, whose P is a bf16 pair
      // (hi in the block's first 32 columns, lo in the next 32): both multiply V
      auto issue_pv = [&](int idx, bool hi_lo) -> bool {
        const int pb = idx & 1, slot = idx % NSV;
        if (!wwait(bar_pfull(mu, pb), (idx >> 1) & 1)) return false;
        if (!wwait(bar_vfull(mu, slot), (idx / NSV) & 1)) return false;
        tc_fence_after();
        const uint64_t dV = smem_desc(sV(mu, slot), 64 * 128, 1024, kSwz128);  // 16 V rows: +2048 B
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(tU + 128, tU + pb * 64 + kk * 8, dV + kk * 128, kIdPV, (idx > 0 || kk > 0) ? 1u : 0u);
        if (C::kHyb && hi_lo) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tU + 128, tU + pb * 64 + 32 + kk * 8, dV + kk * 128, kIdPV, 1u);
        }
        mma_commit_e(bar_ofull(mu));
        mma_commit_e(bar_vfree(mu, slot));
        return true;
      };
      if (ok) {
        int nk = 0;  // this unit's K ring fills consumed so far
        int i = 0;   // entries of this unit issued so far
        bool hyb_prev = false;  // entry i - 1 reads the mixed operands
        auto c = unit_stream<C>(p, mu ? un1 : un0);
        int kt, p0, p1;
        while (c.next(kt, p0, p1)) {
          if (((p0 == TRA_PREC_INT4 || p1 == TRA_PREC_INT4) && !int4) ||
              (!C::kHasF8 && (p0 == TRA_PREC_FP8 || p1 == TRA_PREC_FP8)) ||
              kt > unit_kt_max(mu ? un1 : un0)) {
            *err = TRA_DEV_BAD_LIST;
            ok = false;
            break;
          }
          // S buffer i & 1 last held entry i-2, whose P V this thread has already
          // issued; MMAs of one thread run in order, so QK(i) cannot overtake it
          const uint32_t tSb = tU + (i & 1) * 64;
          const int nf = entry_fills(p0, p1);
          for (int f = 0; f < nf; ++f) {
            const int prec = entry_fill_prec(p0, p1, f);
            const int s = nk % NSK;
            if (!wwait(bar_kfull(mu, s), (uint32_t)((nk / NSK) & 1))) { ok = false; break; }
            tc_fence_after();
            // lanes written: all for a single-precision entry; for two precisions the
            // first MMA writes q-tile 2j's lanes 0-63, the second q-tile 2j+1's 64-127
            const uint32_t keep = nf == 1 ? 0u : 0xFFFFFFFFu;
            const uint32_t msk[4] = {f == 1 ? keep : 0u, f == 1 ? keep : 0u, f == 0 ? keep : 0u,
                                     f == 0 ? keep : 0u};
            const uint32_t kb = sK(mu, s);
            if (C::kHasBf16 && (prec == TRA_PREC_BF16 || prec == kPrecHyb)) {
              // 16 elements of K per MMA: 32 bytes within a 128-byte slab, slabs of 128
              // Q rows (16 KB) and 64 K rows (8 KB)
              const uint64_t dK = smem_desc(kb, 16, 1024, kSwz128);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk)
                mma_bf16_mask(tSb, dQb + (kk >> 2) * 1024 + (kk & 3) * 2, dK + (kk >> 2) * 512 + (kk & 3) * 2,
                              kIdQK16, kk > 0 ? 1u : 0u, msk);
            } else if (C::kHasF8 && prec == TRA_PREC_FP8) {
              // E4M3 x E4M3 -> fp32; operands laid out like the int8 codes (32 bytes of K
              // per MMA)
              const uint64_t dK = smem_desc(kb, 16, C::kI8Sbo, C::kI8Layout);
#pragma unroll
              for (int kk = 0; kk < D / 32; ++kk)
                mma_f8_mask(tSb, dQf + kk * 2, dK + kk * 2, kIdF8, kk > 0 ? 1u : 0u, msk);
            } else {
              const uint64_t dA = prec == TRA_PREC_INT8 ? dQ8 : dQ4;
              const uint64_t dK = smem_desc(kb, 16, C::kI8Sbo, C::kI8Layout);
#pragma unroll
              for (int kk = 0; kk < D / 32; ++kk)
                mma_i8_mask(tSb, dA + kk * 2, dK + kk * 2, kIdI8, kk > 0 ? 1u : 0u, msk);
            }
            mma_commit_e(bar_kfree(mu, s));
            ++nk;
          }
          if (!ok) break;
          mma_commit_e(bar_sfull(mu, i & 1));
          if (i >= 1 && !issue_pv(i - 1, hyb_prev)) { ok = false; break; }
          hyb_prev = p0 == kPrecHyb || p1 == kPrecHyb;
          ++i;
        }
        if (ok && i >= 1 && issue_pv(i - 1, hyb_prev)) mma_commit_e(bar_ofinal(mu));
      }
      // every MMA of this warp completes before TMEM is released
      mma_commit_e(bar_done);
      mbar_wait_drain(bar_done, 0);
      __syncwarp();
    }
  } else if (warp >= 4 && warp < 12) {
    // ================================================================ softmax / epilogue
    const int u = (warp - 4) >> 2;               // unit of this warpgroup
    const Unit x = unit_of(u);
    const int r = (threadIdx.x - 128) & 127;     // query row of the unit = TMEM lane
    const int q4 = warp & 3;                     // TMEM lane quarter of this warp
    const int half = r >> 6, rr = r & 63;        // q-tile of the row (uniform per warp)
    const int qt = x.qt0 + half;
    const bool half_valid = x.valid && qt < x.nt;
    const int tq = qt * kTile + rr;              // query position in the sequence
    const bool row_valid = half_valid && tq < x.T;
    const long long qtile = (long long)x.h * p.ntiles + x.toff + qt;
    const float sq8 = (half_valid && !C::kHyb) ? __ldg(p.sq8 + qtile) : 0.0f;
    // INT4 operands are 16 x code, so INT4 accumulators are 256 x the code product:
    // the power of two goes into the row's INT4 scale (exact)
    const float sq4 = (half_valid && int4) ? __ldg(p.sq4 + qtile) * (1.0f / 256.0f) : 0.0f;
    const float sqf = (half_valid && C::kHasF8) ? __ldg(p.sqf + qtile) : 0.0f;
    const uint32_t lane_addr = ((uint32_t)(q4 * 32) << 16) + (uint32_t)(u * 256);
    const uint32_t tU = tmem + lane_addr, tO = tU + 128;  // S/P buffer b at tU + 64 * b
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    int i = 0;
    auto c = unit_stream<C>(p, x);
    // the K-tile scale of this row's precision of an entry (1 for BF16), loaded one
    // entry ahead (an out-of-range kt, reported by the producer, reads the last
    // in-range tile's scale instead of memory past the sequence)
    const int kt_max = unit_kt_max(x);
    auto kscale = [&](int kt_, int pr) -> float {
      const long long t_ = (long long)x.kvh * p.ntiles + x.toff + min(kt_, kt_max);
      if (pr == TRA_PREC_INT8) return __ldg(p.sk8 + t_);
      if (pr == TRA_PREC_INT4 && int4) return __ldg(p.sk4 + t_);
      if (C::kHyb && pr == kPrecHyb) return __ldg(p.sk4 + t_);
      if (C::kHasF8 && pr == TRA_PREC_FP8) return __ldg(p.skf + t_);
      return 1.0f;
    };
    // hybrid entries: the tile's V INT4 scale and its 64-bit selection mask
    auto hyb_tile = [&](int kt_, int pr, float& sv, uint2& sel) {
      sv = 1.0f;
      sel = make_uint2(0u, 0u);
      if (C::kHyb && pr == kPrecHyb) {
        const long long t_ = (long long)x.kvh * p.ntiles + x.toff + min(kt_, kt_max);
        sv = __ldg(p.sv4 + t_);
        sel = __ldg(reinterpret_cast<const uint2*>(p.sel_mask) + t_);
      }
    };
    int nkt = 0, np0 = 0, np1 = 0;
    bool have = c.next(nkt, np0, np1);
    float nsk = have ? kscale(nkt, half ? np1 : np0) : 0.0f;
    float nsv = 1.0f;
    uint2 nsel = make_uint2(0u, 0u);
    if (C::kHyb && have) hyb_tile(nkt, half ? np1 : np0, nsv, nsel);
    for (; have; ++i) {
      const int kt = nkt, pa = np0, pb = np1;
      const float skt = nsk;
      const float svt = nsv;
      const uint2 selt = nsel;
      have = c.next(nkt, np0, np1);  // look-ahead: next entry and its scale
      if (have) nsk = kscale(nkt, half ? np1 : np0);
      if (C::kHyb && have) hyb_tile(nkt, half ? np1 : np0, nsv, nsel);
      const int sb = i & 1;
      const uint32_t tS = tU + sb * 64;
      if (!mbar_wait(bar_sfull(u, sb), (i >> 1) & 1, err)) { ok = false; break; }
      if (((pa == TRA_PREC_INT4 || pb == TRA_PREC_INT4) && !int4) ||
          (!C::kHasF8 && (pa == TRA_PREC_FP8 || pb == TRA_PREC_FP8)) || kt > kt_max) {
        *err = TRA_DEV_BAD_LIST;
        ok = false;
        break;
      }
      const int prec = half ? pb : pa;  // this row's precision (0: its q-tile skips kt)
      // A q-tile that does not list this tile adds P = 0: its warps skip the TMEM
      // read and every exponential.
      const bool half_applies = prec != 0 && half_valid;
      uint32_t pk[32];
      bool warp_rescale_o = false;
      bool p_stored = false;  // a mixed-operand entry stores its P itself
      float alpha = 1.0f;
      if (!half_applies) {
#pragma unroll
        for (int k = 0; k < 32; ++k) pk[k] = 0u;
      } else {
        tc_fence_after();
        // S in two halves.  Hybrid prefill: columns 32-63 load while columns 0-31 take
        // their per-column selection work (every reader of sr[32..63] waits for the
        // second load first; where both loads are already waited for, that wait is
        // a no-op).  The routed modes gained nothing from the split and wait once.
        uint32_t sr[64];
        {
          uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
          uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
          tmem_ld32(tS, lo);
          if (C::kHyb) {
            tmem_wait_ld();
            tmem_reg_fence(lo);
          }
          tmem_ld32(tS + 32, hi);
          if (!C::kHyb) {
            tmem_wait_ld();
            tmem_reg_fence(lo);
            tmem_reg_fence(hi);
          }
        }
        uint32_t (&s_hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        if (!C::kHyb && p.n_dump > 0) {
          tmem_wait_ld();
          tmem_reg_fence(s_hi);
        }
        if (!C::kHyb && p.n_dump > 0 && row_valid && (prec == TRA_PREC_INT8 || prec == TRA_PREC_INT4)) {
          for (int di = 0; di < p.n_dump; ++di) {
            const int* dc = p.dump_coords + di * 4;
            if (__ldg(dc) == x.b && __ldg(dc + 1) == x.h && __ldg(dc + 2) == qt &&
                __ldg(dc + 3) == kt) {
              int32_t* dst = p.dump_out + ((long long)di * 64 + rr) * 64;
              const int sh = prec == TRA_PREC_INT4 ? 8 : 0;  // INT4: 256 x the code product
              for (int cc = 0; cc < 64; ++cc) dst[cc] = (int32_t)sr[cc] >> sh;
            }
          }
        }
        // log2-domain score = raw * f
        const float f = p.scale_log2 * skt *
                        (prec == TRA_PREC_INT8 ? sq8
                         : prec == TRA_PREC_INT4 ? sq4
                         : (C::kHasF8 && prec == TRA_PREC_FP8) ? sqf : 1.0f);
        // valid keys of this tile for this row, columns [clo, nvalid): causal and
        // sequence end; only the diagonal tile and a sequence's last tile have fewer
        // than 64.  Hybrid: a kPrecHyb entry keeps the keys at least `window`
        // positions behind the query, a BF16 entry the causal keys closer than that.
        int clo = 0;
        int nvalid = row_valid ? min(min(tq - kt * kTile + 1, x.T - kt * kTile), kTile) : 0;
        if (C::kHyb && row_valid) {
          const int behind = tq - kt * kTile;  // query position minus the tile's first key
          if (prec == kPrecHyb)
            nvalid = min(min(behind - p.window + 1, x.T - kt * kTile), kTile);
          else
            clo = max(0, behind - p.window + 1);
        }
        const bool full = __all_sync(0xffffffffu, clo == 0 && nvalid >= kTile);
        // One row of the tile -> bf16 P and the online-softmax update.  Full
        // tiles (every key valid) take a copy with no per-column test; only
        // the diagonal tile and a sequence's last tile take the masked copy.
        // Raw scores as floats: fp32 accumulators as they are, int32 ones
        // converted (exact: |S| < 2^24).  A mode whose tiles are all integer
        // (kInt) takes the row max on the raw int32 values; where fp32 and int32
        // tiles alternate, both share one body (is_int selects the conversion),
        // which keeps the softmax's hot code in one piece.
        auto softmax_row = [&](auto int_tag, auto full_tag, bool is_int) {
          constexpr bool kInt = decltype(int_tag)::value;
          constexpr bool kFull = decltype(full_tag)::value;
          float xs[64];
          // integer row max on the raw accumulators (kInt), else on the converted scores
          int mi4[4];
          float mx4[4];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if (hf == 1) {  // columns 32-63 are in
              tmem_wait_ld();
              tmem_reg_fence(s_hi);
            }
            const int c0 = 32 * hf;
            if (kInt || is_int) {
#pragma unroll
              for (int cc = c0; cc < c0 + 32; ++cc) xs[cc] = (float)(int)sr[cc];
            } else {
#pragma unroll
              for (int cc = c0; cc < c0 + 32; ++cc) xs[cc] = __uint_as_float(sr[cc]);
            }
#pragma unroll
            for (int cc = c0; cc < c0 + 32; ++cc)
              if (!kFull) xs[cc] = (cc >= clo && cc < nvalid) ? xs[cc] : -INFINITY;
            if (kInt && kFull) {
#pragma unroll
              for (int cc = c0; cc < c0 + 32; cc += 8) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  mi4[k] = cc == 0 ? max((int)sr[k], (int)sr[k + 4])
                                   : __vimax3_s32(mi4[k], (int)sr[cc + k], (int)sr[cc + k + 4]);
              }
            } else {
#pragma unroll
              for (int cc = c0; cc < c0 + 32; cc += 8) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  mx4[k] = cc == 0 ? fmaxf(xs[k], xs[k + 4])
                                   : fmaxf(mx4[k], fmaxf(xs[cc + k], xs[cc + k + 4]));
              }
            }
          }
          const float mx = kInt && kFull ? (float)max(max(mi4[0], mi4[1]), max(mi4[2], mi4[3]))
                                         : fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
          const float m_tile = mx == -INFINITY ? -INFINITY : mx * f;  // f > 0 keeps the argmax
          const float m_new = fmaxf(m_run, m_tile);
          const bool need = m_new > m_run + kRescaleThreshold;  // also true for the first finite max
          // once one row of the warp passes the threshold, every row whose max grew
          // moves it too (one O pass for the warp); O is rescaled if one of those rows
          // had seen keys (O rows that have seen none are exactly zero; the rows of a
          // warp may meet their first keys in different entries)
          const bool warp_need = __any_sync(0xffffffffu, need);
          const bool grew = __any_sync(0xffffffffu, m_new > m_run && m_run != -INFINITY);
          warp_rescale_o = warp_need && grew;
          if (warp_need && m_new > m_run) {
            alpha = ex2(m_run - m_new);  // m_run = -inf gives 0
            m_run = m_new;
          }
          // P in bf16 for the MMA; l sums the same bf16-rounded values, so the
          // normalisation matches what P V accumulates.  Packed fp32x2 FMA/add.
          const float2 f2 = make_float2(f, f), nm2 = make_float2(-m_run, -m_run);
          float2 ls[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) ls[k] = make_float2(0.0f, 0.0f);
#pragma unroll
          for (int cc = 0; cc < 64; cc += 2) {
            const float2 arg = __ffma2_rn(make_float2(xs[cc], xs[cc + 1]), f2, nm2);
            float q0 = ex2(arg.x);
            float q1 = ex2(arg.y);
            if (!kFull) {  // masked columns of a row whose max is still -inf
              q0 = (cc >= clo && cc < nvalid) ? q0 : 0.0f;
              q1 = (cc + 1 >= clo && cc + 1 < nvalid) ? q1 : 0.0f;
            }
            const __nv_bfloat162 pbf = __floats2bfloat162_rn(q0, q1);
            const uint32_t w = *reinterpret_cast<const uint32_t*>(&pbf);
            ls[(cc >> 1) & 3] = __fadd2_rn(
                ls[(cc >> 1) & 3],
                make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
            pk[cc >> 1] = w;
          }
          const float2 l2 = __fadd2_rn(__fadd2_rn(ls[0], ls[1]), __fadd2_rn(ls[2], ls[3]));
          l_run = l_run * alpha + (l2.x + l2.y);
        };
        // A hybrid entry (mixed operands): column c of the tile is a selected token's
        // bf16 key (log2 factor f) or an INT4 code row (factor f * sK), and P V
        // reads that token's bf16 V row (P as is) or its INT4 code row (P * sV).
        // An all-zero V tile (sV = 0) has codes 0: its P * sV = 0 adds nothing, as it
        // should, while l still counts p.
        auto hyb_row = [&](auto full_tag) {
          constexpr bool kFull = decltype(full_tag)::value;
          const float fs = p.scale_log2, fc = p.scale_log2 * skt;
          float xs[64];
#pragma unroll
          for (int cc = 0; cc < 64; ++cc) {
            if (cc == 32) {  // columns 32-63 are in
              tmem_wait_ld();
              tmem_reg_fence(s_hi);
            }
            const bool sel = (((cc < 32 ? selt.x : selt.y) >> (cc & 31)) & 1u) != 0u;
            xs[cc] = __uint_as_float(sr[cc]) * (sel ? fs : fc);
            if (!kFull) xs[cc] = (cc >= clo && cc < nvalid) ? xs[cc] : -INFINITY;
          }
          float mx4[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) mx4[k] = fmaxf(xs[k], xs[k + 4]);
#pragma unroll
          for (int cc = 8; cc < 64; cc += 8) {
#pragma unroll
            for (int k = 0; k < 4; ++k) mx4[k] = fmaxf(mx4[k], fmaxf(xs[cc + k], xs[cc + k + 4]));
          }
          const float m_tile = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
          const float m_new = fmaxf(m_run, m_tile);
          const bool need = m_new > m_run + kRescaleThreshold;
          const bool warp_need = __any_sync(0xffffffffu, need);
          const bool grew = __any_sync(0xffffffffu, m_new > m_run && m_run != -INFINITY);
          warp_rescale_o = warp_need && grew;
          if (warp_need && m_new > m_run) {
            alpha = ex2(m_run - m_new);
            m_run = m_new;
          }
          // l adds what P V accumulates, divided by the column's factor: the bf16 P of
          // a selected column, bf16(p * sV) / sV of a code column (an all-zero V tile,
          // sV = 0, takes factor 1: its codes are 0)
          // P written as a bf16 pair hi + lo (lo = the rounding residual of hi), hi in
          // the S block's first 32 columns and lo in the next 32, two halves at a time
          // in pk; P V adds both, so P carries about 16 bits and l sums fp32 p
          float2 ls = make_float2(0.0f, 0.0f);
          // the mask through an opaque copy: the bit tests are recomputed here instead
          // of 64 results being kept live from the score loop (they do not fit)
          uint32_t sw0, sw1;
          asm volatile("mov.b32 %0, %1;" : "=r"(sw0) : "r"(selt.x));
          asm volatile("mov.b32 %0, %1;" : "=r"(sw1) : "r"(selt.y));
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
            for (int cc = 32 * hh; cc < 32 * hh + 32; cc += 2) {
              float q0 = ex2(xs[cc] - m_run);
              float q1 = ex2(xs[cc + 1] - m_run);
              if (!kFull) {
                q0 = (cc >= clo && cc < nvalid) ? q0 : 0.0f;
                q1 = (cc + 1 >= clo && cc + 1 < nvalid) ? q1 : 0.0f;
              }
              ls = __fadd2_rn(ls, make_float2(q0, q1));
              const uint32_t w = cc < 32 ? sw0 : sw1;
              const float g0 = ((w >> (cc & 31)) & 1u) ? q0 : q0 * svt;
              const float g1 = ((w >> ((cc + 1) & 31)) & 1u) ? q1 : q1 * svt;
              const __nv_bfloat162 hb = __floats2bfloat162_rn(g0, g1);
              const uint32_t hw = *reinterpret_cast<const uint32_t*>(&hb);
              const __nv_bfloat162 lb = __floats2bfloat162_rn(g0 - __uint_as_float(hw << 16),
                                                              g1 - __uint_as_float(hw & 0xFFFF0000u));
              pk[((cc >> 1) & 15)] = hw;
              pk[16 + ((cc >> 1) & 15)] = *reinterpret_cast<const uint32_t*>(&lb);
            }
            tmem_st16(tS + 16 * hh, *reinterpret_cast<const uint32_t(*)[16]>(&pk[0]));
            tmem_st16(tS + 32 + 16 * hh, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16]));
          }
          l_run = l_run * alpha + (ls.x + ls.y);
        };
        using T_ = std::true_type;
        using F_ = std::false_type;
        if (C::kHyb && prec == kPrecHyb) {
          if (full) hyb_row(T_{}); else hyb_row(F_{});
          p_stored = true;
        } else if (C::kFloatScores) {
          const bool is_int = !(prec == TRA_PREC_BF16 || (C::kHasF8 && prec == TRA_PREC_FP8));
          if (full) softmax_row(F_{}, T_{}, is_int); else softmax_row(F_{}, F_{}, is_int);
        } else {
          if (full) softmax_row(T_{}, T_{}, true); else softmax_row(T_{}, F_{}, true);
        }
      }
      if (warp_rescale_o && i >= 1) {
        // rescaling O needs every earlier P V complete.  sfull(i) already implies
        // P V(<= i-2) complete (they were issued before QK(i)), so ofull is at
        // phase i-1 or i and the parity wait below is exact.
        if (!mbar_wait(bar_ofull(u), (i - 1) & 1, err)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int col = 0; col < D; col += 32) {
          uint32_t o[32];
          tmem_ld32(tO + col, o);
          tmem_wait_ld();
          tmem_reg_fence(o);
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(tO + col, o);
        }
      }
      if (!p_stored) {
        tmem_st32(tS, pk);  // P(i) over S(i), which this thread has read
        // a mixed-operand entry's P V also reads the lo half: zero for these rows too
        if (C::kHyb && (pa == kPrecHyb || pb == kPrecHyb)) tmem_st32(tS + 32, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_pfull(u, sb));
    }
    // ---- epilogue: O / l
    // (a parity wait on ofull could pass one phase early here, so the epilogue
    // waits for the unit's final commit instead)
    if (ok && i > 0 && mbar_wait(bar_ofinal(u), 0, err)) {
      tc_fence_after();
      const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      uint16_t* orow = p.out + ((long long)(x.seq0 + tq) * p.Hq + x.h) * D;
#pragma unroll 1
      for (int col = 0; col < D; col += 32) {
        uint32_t o[32];
        tmem_ld32(tO + col, o);
        tmem_wait_ld();
        tmem_reg_fence(o);
        if (row_valid) {
#pragma unroll
          for (int k = 0; k < 32; k += 8) {
            uint32_t w[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              const __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(o[k + 2 * y]) * inv,
                                                              __uint_as_float(o[k + 2 * y + 1]) * inv);
              w[y] = *reinterpret_cast<const uint32_t*>(&v2);
            }
            *reinterpret_cast<uint4*>(orow + col + k) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (row_valid && p.lse)
        p.lse[(long long)x.h * __ldg(p.cu + p.B) + x.seq0 + tq] =
            (m_run + __log2f(l_run)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
  if (threadIdx.x == 0 && *err) atomicOr(p.status, *err);
}

// the launch parameters stay within the classic 4 KB kernel-parameter space
static_assert(sizeof(PrefillParams) + sizeof(PrefillMaps) <= 4096, "prefill launch parameters");

template <int D, int MODE>
cudaError_t launch_one(const PrefillParams& p, const PrefillMaps& m, cudaStream_t s) {
  using C = Cfg<D, MODE>;
  const long long units = (long long)p.jmax * p.B * p.Hq;
  const long long ctas = (units + C::kCtaUnits - 1) / C::kCtaUnits;
  if (ctas == 0) return cudaSuccess;
  if (ctas > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  prefill_kernel<D, MODE><<<(unsigned)ctas, kThreads, C::kSmemBytes, s>>>(p, m);
  return cudaGetLastError();
}

}  // namespace

template <int D>
cudaError_t launch_d(const PrefillParams& p, const PrefillMaps& m, cudaStream_t s) {
  if (p.mode == TRA_POLICY_BITMASK) return launch_one<D, TRA_POLICY_BITMASK>(p, m, s);
  if (p.mode == TRA_POLICY_MIXED) return launch_one<D, TRA_POLICY_MIXED>(p, m, s);
  if (p.mode == kPrefillModeHybrid) return launch_one<D, kPrefillModeHybrid>(p, m, s);
  if (p.mode == kPrefillModeBoundaryF8) return launch_one<D, kPrefillModeBoundaryF8>(p, m, s);
  return launch_one<D, TRA_POLICY_BOUNDARY>(p, m, s);
}

cudaError_t launch_prefill(const PrefillParams& p, const PrefillMaps& m, cudaStream_t s) {
  return p.d == 128 ? launch_d<128>(p, m, s) : launch_d<64>(p, m, s);
}

}  // namespace tra
