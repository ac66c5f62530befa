// prefill.cu -- fused causal prefill attention over precision-grouped tile
// traversals (TriAttention abstract: one fused kernel skips omitted tiles and
// merges both QK precisions into a single normalised output; TileMix abstract:
// each tile group goes through a high-precision or an INT8 score path and both
// paths update the same online-softmax state).
//
// Work unit: one query head h of one sequence b and one pair of q-tiles
// (2j, 2j+1) = 128 query rows, the M of one tcgen05 MMA.  The two rows' CSR
// traversals (each sorted by (precision, kt)) are merged on the fly into one
// stream of (kt, precision, half-mask) entries; an entry whose tile appears in
// only one q-tile's list (or with a different precision) is computed for all
// 128 rows and masked to -inf in the other half, so routing stays exact.
//
// Warp roles (256 threads):
//   warp 0      TMA producer: Q tiles once, then K (INT8 codes or BF16) and V
//               (BF16) tiles into an NST-deep ring;
//   warp 1      TMEM owner and MMA issuer: S = Q K^T with kind::i8 (INT8/INT4,
//               exact int32) or kind::f16 (BF16, fp32) into a double-buffered S
//               in TMEM, then O += P V (bf16) into TMEM;
//   warps 2-3   INT4 expanders: packed INT4 codes (Q once, K per INT4 entry)
//               sign-extended to int8 in the swizzled operand layout (tcgen05
//               has no integer 4-bit MMA, so INT4 tiles run as int8 MMAs);
//   warps 4-7   softmax / epilogue: one thread per query row (TMEM lane):
//               S -> scaled log2 scores -> mask -> online softmax with lazy
//               rescaling of O -> bf16 P in shared memory; finally O / l.
#include "tra_device.cuh"
#include "tra_launch.h"

namespace tra {
namespace {

constexpr int kThreads = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only past 2^8 growth

template <int D, int MODE>
struct Cfg {
  static constexpr int kStages = 4;
  static constexpr int kQ8Bytes = 128 * D;                                    // int8 Q codes
  static constexpr int kQxBytes = MODE == TRA_POLICY_BITMASK ? 128 * D * 2 : 128 * D;
  static constexpr int kKBytes = 64 * D * 2;                                  // slot fits bf16
  static constexpr int kVBytes = 64 * D * 2;
  static constexpr int kPBytes = 128 * 64 * 2;
  static constexpr int kOffQ8 = 0;
  static constexpr int kOffQx = kOffQ8 + kQ8Bytes;
  static constexpr int kOffK = kOffQx + kQxBytes;
  static constexpr int kOffV = kOffK + kStages * kKBytes;
  static constexpr int kOffP = kOffV + kStages * kVBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  static constexpr int kNumBars = 2 + 5 * kStages + 2 + 2 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
  // int8 K-major rows of D bytes: 128-byte swizzle for D = 128, 64-byte for D = 64
  static constexpr uint32_t kI8Layout = D == 128 ? kSwz128 : kSwz64;
  static constexpr uint32_t kI8Sbo = D == 128 ? 1024 : 512;
  static constexpr int kSlabs = D / 64;  // bf16 64-element (128-byte) slabs per row
};

// Byte offset of 16-byte chunk `c` of row `r` in a swizzled K-major int8 tile.
template <int D>
__device__ __forceinline__ uint32_t i8_swz_offset(int r, int c) {
  if (D == 128) return r * 128 + ((c ^ (r & 7)) << 4);
  return r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
}

// Merge of two sorted CSR rows (entry = (prec << 28) | kt): yields each
// distinct entry once with a mask of the rows (bit 0: first, bit 1: second)
// that contain it.
struct MergeCursor {
  const uint32_t* e;
  int p0, e0, p1, e1;
  __device__ __forceinline__ bool next(uint32_t& val, int& mask) {
    const uint32_t a = p0 < e0 ? __ldg(e + p0) : 0xFFFFFFFFu;
    const uint32_t b = p1 < e1 ? __ldg(e + p1) : 0xFFFFFFFFu;
    if (a == 0xFFFFFFFFu && b == 0xFFFFFFFFu) return false;
    if (a < b) {
      val = a; mask = 1; ++p0;
    } else if (b < a) {
      val = b; mask = 2; ++p1;
    } else {
      val = a; mask = 3; ++p0; ++p1;
    }
    return true;
  }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ PrefillMaps m) {
  using C = Cfg<D, MODE>;
  constexpr int NST = C::kStages;
  extern __shared__ uint8_t smem_raw[];

  // ---- work unit: heaviest q-tile pairs first, heads fastest
  const int h = blockIdx.x % p.Hq;
  const int b = (blockIdx.x / p.Hq) % p.B;
  const int j = p.jmax - 1 - (int)(blockIdx.x / (p.Hq * p.B));
  const int seq0 = __ldg(p.cu + b);
  const int T = __ldg(p.cu + b + 1) - seq0;
  const int nt = (T + kTile - 1) / kTile;
  if (2 * j >= nt) return;  // uniform exit, before any barrier or TMEM use
  const int toff = seq_tile_offset(p.cu, b);
  const int grp = p.Hq / p.Hkv;
  const int kvh = h / grp;
  const int qt0 = 2 * j;
  const bool has_second = qt0 + 1 < nt;
  // INT4 operands exist only for boundary policies with an INT4 region; a list
  // entry asking for INT4 without them is reported, never read
  const bool int4 = MODE == TRA_POLICY_BOUNDARY && p.has_int4;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - smem_u32(smem_raw));
  const uint32_t sQ8 = base + C::kOffQ8;
  const uint32_t sQx = base + C::kOffQx;
  const uint32_t sK = base + C::kOffK;
  const uint32_t sV = base + C::kOffV;
  const uint32_t sP = base + C::kOffP;
  const uint32_t bars = base + C::kOffBar;
  const uint32_t bar_q = bars + 0 * 8;
  const uint32_t bar_q4 = bars + 1 * 8;
  auto bar_kfull = [&](int s) { return bars + (2 + s) * 8; };
  auto bar_k4full = [&](int s) { return bars + (2 + NST + s) * 8; };
  auto bar_kfree = [&](int s) { return bars + (2 + 2 * NST + s) * 8; };
  auto bar_vfull = [&](int s) { return bars + (2 + 3 * NST + s) * 8; };
  auto bar_vfree = [&](int s) { return bars + (2 + 4 * NST + s) * 8; };
  auto bar_sfull = [&](int s) { return bars + (2 + 5 * NST + s) * 8; };
  auto bar_sfree = [&](int s) { return bars + (4 + 5 * NST + s) * 8; };
  const uint32_t bar_pfull = bars + (6 + 5 * NST) * 8;
  const uint32_t bar_ofull = bars + (7 + 5 * NST) * 8;
  const uint32_t bar_done = bars + (8 + 5 * NST) * 8;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::kOffMisc);
  volatile int* const err = reinterpret_cast<volatile int*>(gbase + C::kOffMisc + 16);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_q4, 64);
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_k4full(s), 64);
      mbar_init(bar_kfree(s), 1);
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_vfree(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_sfull(s), 1);
      mbar_init(bar_sfree(s), 128);
    }
    mbar_init(bar_pfull, 128);
    mbar_init(bar_ofull, 1);
    mbar_init(bar_done, 1);
    *err = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int row0 = h * p.ntiles + toff + qt0;
  MergeCursor cur0;
  cur0.e = p.entries;
  cur0.p0 = __ldg(p.row_ptr + row0);
  cur0.e0 = __ldg(p.row_ptr + row0 + 1);
  cur0.p1 = cur0.e0;
  cur0.e1 = has_second ? __ldg(p.row_ptr + row0 + 2) : cur0.e0;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint32_t qbytes = C::kQ8Bytes + (MODE == TRA_POLICY_BITMASK ? 128 * D * 2 : 0);
      mbar_arrive_expect_tx(bar_q, qbytes);
      tma_load_2d(sQ8, &m.q8, bar_q, 0, row0 * kTile);
      if (MODE == TRA_POLICY_BITMASK) {
        for (int sl = 0; sl < C::kSlabs; ++sl)
          tma_load_3d(sQx + sl * 128 * 128, &m.qb, bar_q, sl * 64, h, seq0 + qt0 * kTile);
      }
      MergeCursor c = cur0;
      uint32_t val;
      int mask;
      for (int i = 0; c.next(val, mask); ++i) {
        const int s = i % NST, use = i / NST;
        const uint32_t prec = val >> 28;
        const int kt = (int)(val & 0x0FFFFFFFu);
        if (prec == TRA_PREC_INT4 && !int4) {
          *err = TRA_DEV_BAD_LIST;
          break;
        }
        if (prec != TRA_PREC_INT4) {
          if (use > 0 && !mbar_wait(bar_kfree(s), (use - 1) & 1, err)) break;
          const uint32_t dst = sK + s * C::kKBytes;
          if (prec == TRA_PREC_INT8) {
            mbar_arrive_expect_tx(bar_kfull(s), 64 * D);
            tma_load_2d(dst, &m.k8, bar_kfull(s), 0, (kvh * p.ntiles + toff + kt) * kTile);
          } else {
            mbar_arrive_expect_tx(bar_kfull(s), 64 * D * 2);
            for (int sl = 0; sl < C::kSlabs; ++sl)
              tma_load_3d(dst + sl * 64 * 128, &m.kb, bar_kfull(s), sl * 64, kvh, seq0 + kt * kTile);
          }
        }
        if (use > 0 && !mbar_wait(bar_vfree(s), (use - 1) & 1, err)) break;
        mbar_arrive_expect_tx(bar_vfull(s), 64 * D * 2);
        for (int sl = 0; sl < C::kSlabs; ++sl)
          tma_load_3d(sV + s * C::kVBytes + sl * 64 * 128, &m.vb, bar_vfull(s), sl * 64, kvh,
                      seq0 + kt * kTile);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdI8 = instr_desc(2, 1, 0, 0, 64, 128);
      constexpr uint32_t kIdQK16 = instr_desc(1, 1, 0, 0, 64, 128);
      constexpr uint32_t kIdPV = instr_desc(1, 1, 0, 1, D, 128);
      const uint32_t tS = tmem, tO = tmem + 128;
      bool ok = mbar_wait(bar_q, 0, err);
      if (ok && int4) ok = mbar_wait(bar_q4, 0, err);
      tc_fence_after();
      uint32_t kph = 0, k4ph = 0;  // per-slot phase bits of kfull / k4full
      auto issue_pv = [&](int jj) -> bool {
        const int s = jj % NST;
        if (!mbar_wait(bar_pfull, jj & 1, err)) return false;
        if (!mbar_wait(bar_vfull(s), (jj / NST) & 1, err)) return false;
        tc_fence_after();
        const uint32_t vb = sV + s * C::kVBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t a = smem_desc(sP + kk * 32, 16, 1024, kSwz128);
          const uint64_t bd = smem_desc(vb + kk * 2048, 64 * 128, 1024, kSwz128);
          mma_bf16(tO, a, bd, kIdPV, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_ofull);
        mma_commit(bar_vfree(s));
        return true;
      };
      int i = 0;
      if (ok) {
        MergeCursor c = cur0;
        uint32_t val;
        int mask;
        for (; c.next(val, mask); ++i) {
          const int s = i % NST, buf = i & 1;
          const uint32_t prec = val >> 28;
          if (prec == TRA_PREC_INT4 && !int4) {
            *err = TRA_DEV_BAD_LIST;
            ok = false;
            break;
          }
          if (prec == TRA_PREC_INT4) {
            ok = mbar_wait(bar_k4full(s), (k4ph >> s) & 1, err);
            k4ph ^= 1u << s;
          } else {
            ok = mbar_wait(bar_kfull(s), (kph >> s) & 1, err);
            kph ^= 1u << s;
          }
          if (ok && i >= 2) ok = mbar_wait(bar_sfree(buf), ((i >> 1) - 1) & 1, err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = sK + s * C::kKBytes;
          const uint32_t dS = tS + buf * 64;
          if (prec == TRA_PREC_BF16) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const int sl = kk >> 2, off = (kk & 3) * 32;
              const uint64_t a = smem_desc(sQx + sl * 128 * 128 + off, 16, 1024, kSwz128);
              const uint64_t bd = smem_desc(kb + sl * 64 * 128 + off, 16, 1024, kSwz128);
              mma_bf16(dS, a, bd, kIdQK16, kk > 0 ? 1u : 0u);
            }
          } else {
            const uint32_t qa = prec == TRA_PREC_INT8 ? sQ8 : sQx;
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) {
              const uint64_t a = smem_desc(qa + kk * 32, 16, C::kI8Sbo, C::kI8Layout);
              const uint64_t bd = smem_desc(kb + kk * 32, 16, C::kI8Sbo, C::kI8Layout);
              mma_i8(dS, a, bd, kIdI8, kk > 0 ? 1u : 0u);
            }
          }
          mma_commit(bar_sfull(buf));
          mma_commit(bar_kfree(s));
          if (i >= 1 && !issue_pv(i - 1)) { ok = false; break; }
        }
        if (ok && i >= 1) issue_pv(i - 1);
      }
      // all MMAs issued by this thread complete before TMEM is released
      mma_commit(bar_done);
      mbar_wait(bar_done, 0, err);
    }
  } else if (warp == 2 || warp == 3) {
    // ================================================================ INT4 expanders
    const int t = threadIdx.x - 64;  // 0..63
    constexpr int kPackedRow = D / 2;          // bytes per packed row
    constexpr int kChunksPerRow = kPackedRow / 16;
    bool ok = true;
    if (int4) {
      // Q: 128 rows (two q-tiles); rows of a missing second q-tile stay zero
      const uint8_t* src = p.q4 + (long long)row0 * kTile * kPackedRow;
      const int rows = has_second ? 128 : 64;
      for (int f = t; f < 128 * kChunksPerRow; f += 64) {
        const int r = f / kChunksPerRow, c = f % kChunksPerRow;
        uint4 w = make_uint4(0, 0, 0, 0);
        if (r < rows) w = __ldg(reinterpret_cast<const uint4*>(src + r * kPackedRow + c * 16));
        const uint2 e0 = expand_int4x8(w.x), e1 = expand_int4x8(w.y);
        const uint2 e2 = expand_int4x8(w.z), e3 = expand_int4x8(w.w);
        uint8_t* dst = gbase + C::kOffQx;
        *reinterpret_cast<uint4*>(dst + i8_swz_offset<D>(r, 2 * c)) = make_uint4(e0.x, e0.y, e1.x, e1.y);
        *reinterpret_cast<uint4*>(dst + i8_swz_offset<D>(r, 2 * c + 1)) = make_uint4(e2.x, e2.y, e3.x, e3.y);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_q4);
      MergeCursor c = cur0;
      uint32_t val;
      int mask;
      for (int i = 0; c.next(val, mask); ++i) {
        if ((val >> 28) != TRA_PREC_INT4) continue;
        const int s = i % NST, use = i / NST;
        if (use > 0 && !mbar_wait(bar_kfree(s), (use - 1) & 1, err)) { ok = false; break; }
        const int kt = (int)(val & 0x0FFFFFFFu);
        const uint8_t* ks = p.k4 + ((long long)(kvh * p.ntiles + toff + kt) * kTile) * kPackedRow;
        uint8_t* dst = gbase + C::kOffK + s * C::kKBytes;
        for (int f = t; f < 64 * kChunksPerRow; f += 64) {
          const int r = f / kChunksPerRow, cc = f % kChunksPerRow;
          const uint4 w = __ldg(reinterpret_cast<const uint4*>(ks + r * kPackedRow + cc * 16));
          const uint2 e0 = expand_int4x8(w.x), e1 = expand_int4x8(w.y);
          const uint2 e2 = expand_int4x8(w.z), e3 = expand_int4x8(w.w);
          *reinterpret_cast<uint4*>(dst + i8_swz_offset<D>(r, 2 * cc)) = make_uint4(e0.x, e0.y, e1.x, e1.y);
          *reinterpret_cast<uint4*>(dst + i8_swz_offset<D>(r, 2 * cc + 1)) = make_uint4(e2.x, e2.y, e3.x, e3.y);
        }
        fence_proxy_async_smem();
        mbar_arrive(bar_k4full(s));
      }
    }
    (void)ok;
  } else {
    // ================================================================ softmax / epilogue
    const int r = threadIdx.x - 128;       // query row of the unit = TMEM lane
    const int q4 = warp & 3;               // TMEM lane quarter of this warp
    const int half = r >> 6, rr = r & 63;
    const int qt = qt0 + half;
    const bool half_valid = qt < nt;
    const int tq = qt * kTile + rr;        // query position in the sequence
    const bool row_valid = half_valid && tq < T;
    const long long qtile = (long long)h * p.ntiles + toff + qt;
    const float sq8 = half_valid ? __ldg(p.sq8 + qtile) : 0.0f;
    const float sq4 = (half_valid && int4) ? __ldg(p.sq4 + qtile) : 0.0f;
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    uint8_t* const prow = gbase + C::kOffP + r * 128;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    int i = 0;
    MergeCursor c = cur0;
    uint32_t val;
    int mask;
    for (; c.next(val, mask); ++i) {
      const int buf = i & 1;
      if (!mbar_wait(bar_sfull(buf), (i >> 1) & 1, err)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        tmem_ld32(tmem + lane_addr + buf * 64, lo);
        tmem_ld32(tmem + lane_addr + buf * 64 + 32, hi);
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar_sfree(buf));

      const uint32_t prec = val >> 28;
      const int kt = (int)(val & 0x0FFFFFFFu);
      if (prec == TRA_PREC_INT4 && !int4) {
        *err = TRA_DEV_BAD_LIST;
        ok = false;
        break;
      }
      const bool applies = ((mask >> half) & 1) && row_valid;
      if (p.n_dump > 0 && applies && prec != TRA_PREC_BF16) {
        for (int di = 0; di < p.n_dump; ++di) {
          const int* dc = p.dump_coords + di * 4;
          if (__ldg(dc) == b && __ldg(dc + 1) == h && __ldg(dc + 2) == qt && __ldg(dc + 3) == kt) {
            int32_t* dst = p.dump_out + ((long long)di * 64 + rr) * 64;
            for (int cc = 0; cc < 64; ++cc) dst[cc] = (int32_t)sr[cc];
          }
        }
      }
      const long long ktile = (long long)kvh * p.ntiles + toff + kt;
      float f = p.scale_log2;
      if (prec == TRA_PREC_INT8) f *= sq8 * __ldg(p.sk8 + ktile);
      else if (prec == TRA_PREC_INT4) f *= sq4 * __ldg(p.sk4 + ktile);
      // number of valid keys of this tile for this row (causal and sequence end)
      int nvalid = 0;
      if (applies) nvalid = min(min(tq - kt * kTile + 1, T - kt * kTile), kTile);
      float s[64];
      float m_tile = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < 64; ++cc) {
        const float raw = prec == TRA_PREC_BF16 ? __uint_as_float(sr[cc]) : (float)(int)sr[cc];
        s[cc] = cc < nvalid ? raw * f : -INFINITY;
        m_tile = fmaxf(m_tile, s[cc]);
      }
      const float m_new = fmaxf(m_run, m_tile);
      const bool need = m_new > m_run + kRescaleThreshold;  // also true for the first finite max
      const bool warp_need = __any_sync(0xffffffffu, need);
      float alpha = 1.0f;
      if (warp_need && m_new > m_run) {
        alpha = ex2(m_run - m_new);  // m_run = -inf gives 0
        m_run = m_new;
      }
      float l_tile = 0.0f;
      uint32_t pk[32];
#pragma unroll
      for (int cc = 0; cc < 64; cc += 2) {
        const float p0 = cc < nvalid ? ex2(s[cc] - m_run) : 0.0f;
        const float p1 = cc + 1 < nvalid ? ex2(s[cc + 1] - m_run) : 0.0f;
        const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
        const float2 pr = __bfloat1622float2(pb);
        l_tile += pr.x + pr.y;
        pk[cc >> 1] = *reinterpret_cast<const uint32_t*>(&pb);
      }
      l_run = l_run * alpha + l_tile;
      if (i > 0) {
        if (!mbar_wait(bar_ofull, (i - 1) & 1, err)) { ok = false; break; }
        tc_fence_after();
        if (warp_need) {
#pragma unroll 1
          for (int col = 0; col < D; col += 32) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_addr + 128 + col, o);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
            tmem_st32(tmem + lane_addr + 128 + col, o);
          }
          tmem_wait_st();
        }
      }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        *reinterpret_cast<uint4*>(prow + ((ch ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_pfull);
    }
    // ---- epilogue: O / l
    if (ok && i > 0 && mbar_wait(bar_ofull, (i - 1) & 1, err)) {
      tc_fence_after();
      const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      uint16_t* orow = p.out + ((long long)(seq0 + tq) * p.Hq + h) * D;
#pragma unroll 1
      for (int col = 0; col < D; col += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_addr + 128 + col, o);
        tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int x = 0; x < 32; x += 8) {
            uint32_t w[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              const __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(o[x + 2 * y]) * inv,
                                                              __uint_as_float(o[x + 2 * y + 1]) * inv);
              w[y] = *reinterpret_cast<const uint32_t*>(&v2);
            }
            *reinterpret_cast<uint4*>(orow + col + x) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (row_valid && p.lse)
        p.lse[(long long)h * __ldg(p.cu + p.B) + seq0 + tq] =
            (m_run + __log2f(l_run)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
  if (threadIdx.x == 0 && *err) atomicOr(p.status, *err);
}

template <int D, int MODE>
cudaError_t launch_one(const PrefillParams& p, const PrefillMaps& m, cudaStream_t s) {
  using C = Cfg<D, MODE>;
  const long long ctas = (long long)p.jmax * p.B * p.Hq;
  if (ctas == 0) return cudaSuccess;
  if (ctas > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  prefill_kernel<D, MODE><<<(unsigned)ctas, kThreads, C::kSmemBytes, s>>>(p, m);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams& p, const PrefillMaps& m, cudaStream_t s) {
  if (p.d == 128)
    return p.mode == TRA_POLICY_BITMASK ? launch_one<128, TRA_POLICY_BITMASK>(p, m, s)
                                        : launch_one<128, TRA_POLICY_BOUNDARY>(p, m, s);
  return p.mode == TRA_POLICY_BITMASK ? launch_one<64, TRA_POLICY_BITMASK>(p, m, s)
                                      : launch_one<64, TRA_POLICY_BOUNDARY>(p, m, s);
}

}  // namespace tra
