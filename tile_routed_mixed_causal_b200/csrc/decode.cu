// decode.cu -- one decode step over the compressed KV cache (TriAttention
// abstract: the K/V quantised during prefill become a compressed KV cache for
// decoding, which cuts the re-reading of the prompt; HyQuant, "How HyQuant
// works": dequantisation is done inside the attention kernel so it costs no
// extra memory pass).
//
// Split-K over the cached tiles of each (sequence, KV head).  A CTA is one
// producer warp and four consumer warps.  The producer streams the split's
// kept K/V tiles (INT8 or INT4 codes, one 64-token tile per ring stage) with
// 2-D TMA copies whose 128/64-byte swizzle makes the per-key row reads below
// bank-conflict free.  Each consumer warp takes every fourth tile and keeps its
// own online-softmax state for all query heads of the GQA group, so the loop has
// no block barrier and every cached byte is read once per group:
//   scores: S^T = K Q^T on the tensor cores as integer MMAs (mma.sync m16n8k32,
//           s8 x s8 -> s32): the K codes go in as they are stored (INT4 nibbles
//           masked in place, worth 16 x code), q as a 24-bit fixed-point triple of
//           int8 limbs per head; K tiles fed by ldmatrix;
//   softmax: per head over the warp's fragment lanes, K scale and 1/sqrt(d)
//           folded into the exponent, V scale folded into P (f16, staged per warp);
//   P V:    O^T += V^T P^T on the tensor cores, V fed by ldmatrix.trans.
// The bf16 tail (earlier decode tokens + the new one) goes to the last data split
// of every (sequence, KV head): after its cached tiles, its four warps share the
// tail keys on the CUDA cores, so the grid holds data splits only.  The four warps' states are merged per
// CTA; the last split of each (sequence, KV head) to finish merges the splits
// into the output, and the last such row of a sequence advances tail_len.
#include <type_traits>

#include "tra_device.cuh"
#include "tra_launch.h"

namespace tra {
namespace {

constexpr int kConsumers = 4;
constexpr int kDecThreads = 32 * (kConsumers + 1);
constexpr int kDecStages = 6;
// Two q limbs serve a CTA whose query heads all have max |q| < 2^kTwoLimbMaxE.  Measured
// on a decode cache with x10 outlier K channels, the output error of two limbs against
// exact q stays below about 1e-3 up to there and doubles with every further power of two.
constexpr int kTwoLimbMaxE = 4;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of 16-byte chunk c of row r in a tile whose rows are R bytes,
// written by TMA with an R-byte swizzle (R = 128, 64 or 32).
template <int R>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return r * R + ((c ^ ((r * R >> 7) & (R / 16 - 1))) << 4);
}

// ---------------------------------------------------------------- mma.sync helpers
// The GQA group's contractions run on the tensor cores.  Scores S^T = K Q^T are
// m16n8k32 integer MMAs (M = 16 keys, N = 8 columns of (head, q limb) pairs, exact
// int32 accumulation); O^T += V^T P^T are m16n8k16 MMAs (f16 inputs, fp32
// accumulation; M = 16 channels, N = 8 heads), whose V codes reach f16 exactly:
// each biased byte / nibble becomes the low mantissa byte of 1024.0h, and one
// packed subtraction removes the bias.  ldmatrix on the int8 tiles, viewed as
// 16-bit pairs, hands every thread four consecutive bytes; the k (channel or
// key) order inside an MMA is a permutation applied identically to both operands.

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Four signed INT4 codes of a word's even / odd nibbles as int8 lanes worth
// 16 x code (exact: the nibble becomes the high half of its byte).
__device__ __forceinline__ uint32_t i4_even_x16(uint32_t x) { return (x << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t i4_odd_x16(uint32_t x) { return x & 0xF0F0F0F0u; }
// Two biased bytes (selected by `sel` from x) -> f16x2 of (byte - bias).
__device__ __forceinline__ uint32_t h2_from_bytes(uint32_t x, uint32_t sel, uint32_t bias2) {
  uint32_t h = __byte_perm(x, 0x6464u, sel);
  asm("sub.rn.f16x2 %0, %0, %1;" : "+r"(h) : "r"(bias2));
  return h;
}
// Eight signed INT4 codes of a word (channel i in bits 4i .. 4i+3) -> four exact
// f16x2: channels (0, 4), (1, 5), (2, 6), (3, 7).  One lop3 per pair computes
// (x & mask) ^ magic, which flips the nibble's sign bit (code + 8) and places it
// in the low mantissa bits of 1024.0h (even nibbles) or, scaled by 16, of the
// same (odd nibbles); a packed subtract / fma removes the offset exactly.
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));  // (a & b) ^ c
  return d;
}
__device__ __forceinline__ void i4x8_to_h2(uint32_t x, uint32_t (&h)[4]) {
  const uint32_t y = x >> 8;
  h[0] = and_xor(x, 0x000F000Fu, 0x64086408u);
  h[1] = and_xor(x, 0x00F000F0u, 0x64806480u);
  h[2] = and_xor(y, 0x000F000Fu, 0x64086408u);
  h[3] = and_xor(y, 0x00F000F0u, 0x64806480u);
  const uint32_t bias = 0x64086408u;      // (1032, 1032) = 1024 + 8
  const uint32_t sixteenth = 0x2C002C00u;  // (1/16, 1/16)
  const uint32_t m72 = 0xD480D480u;        // (-72, -72) = -(1024 + 128) / 16
  asm("sub.rn.f16x2 %0, %0, %1;" : "+r"(h[0]) : "r"(bias));
  asm("sub.rn.f16x2 %0, %0, %1;" : "+r"(h[2]) : "r"(bias));
  asm("fma.rn.f16x2 %0, %0, %1, %2;" : "+r"(h[1]) : "r"(sixteenth), "r"(m72));
  asm("fma.rn.f16x2 %0, %0, %1, %2;" : "+r"(h[3]) : "r"(sixteenth), "r"(m72));
}
constexpr uint32_t kSel02 = 0x5240, kSel13 = 0x5341;
constexpr uint32_t kBias8 = 0x64806480u;  // f16x2 (1152, 1152) = 1024 + 128

// Named barrier over the whole CTA, usable from different code locations.
__device__ __forceinline__ void named_sync(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kDecThreads) : "memory");
}

template <int D, int GRP>
struct DecCfg {
  static constexpr int kRow8 = D;                // INT8 row bytes
  static constexpr int kRow4 = D / 2;            // INT4 row bytes
  static constexpr int kTileBytes = kTile * D;   // INT8 codes of one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static_assert(kConsumers <= kDecStages, "the consumers' parity waits need kConsumers <= kDecStages");
  static constexpr int kPStride = 72;            // f16 per head row of P (bank-conflict free)
  static constexpr int kOffQ = kDecStages * kStageBytes;  // q: [D/2 pairs][GRP] float2
  static constexpr int kQBytes = (D / 2) * GRP * 8;
  static constexpr int kOffP = kOffQ + kQBytes;            // P: [warp][8 heads][kPStride] f16
  static constexpr int kPBytes = kConsumers * 8 * kPStride * 2;
  static constexpr int kOffE = kOffP + kPBytes;            // q limb exponents: [GRP] int
  static constexpr int kEBytes = 32;
  static constexpr int kStates = 2 * kConsumers;           // tile + tail state per warp
  // merge area [state][GRP][D + 2] floats, aliasing the drained ring
  static constexpr int kOffRed = 0;
  static constexpr int kRedBytes = kStates * GRP * (D + 2) * 4;
  static_assert(kRedBytes <= kDecStages * kStageBytes, "merge area must fit in the ring");
  static_assert((2 * TRA_MAX_DECODE_SPLITS + 1) * GRP * 4 <= kDecStages * kStageBytes,
                "split weights must fit in the ring");
  static constexpr int kOffBar = kOffE + kEBytes;
  static constexpr int kSmem = kOffBar + 2 * kDecStages * 8 + 16 + 1024;
  static constexpr int kCh = D / 32;             // tail P V channels per lane
  static constexpr int kB8 = D / 16;             // 16-channel blocks of the O fragments
  static constexpr int kQM = GRP > 4 ? 2 : 1;    // (hi, mid) limb MMAs per K fragment (4 heads each)
};

template <int D, int GRP, int NL, bool HYB>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(
    const DecodeParams p, const __grid_constant__ DecodeMaps m) {
  using C = DecCfg<D, GRP>;
  extern __shared__ uint8_t dsm_raw[];
  const uint32_t base = (smem_u32(dsm_raw) + 1023u) & ~1023u;
  uint8_t* const sm = dsm_raw + (base - smem_u32(dsm_raw));
  float2* const q2 = reinterpret_cast<float2*>(sm + C::kOffQ);
  float* const red = reinterpret_cast<float*>(sm + C::kOffRed);
  const uint32_t bar_full = base + C::kOffBar;
  const uint32_t bar_empty = bar_full + kDecStages * 8;
  volatile int* const err =
      reinterpret_cast<volatile int*>(sm + C::kOffBar + 2 * kDecStages * 8);

  // x: data split x of (b, kvh); the last one also attends over the bf16 tail
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int nsplit = p.splits, split = (int)blockIdx.x;
  const bool tail_cta = split == nsplit - 1;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int grp = p.Hq / p.Hkv;
  const int seq0 = __ldg(p.cu + b);
  const int T = __ldg(p.cu + b + 1) - seq0;
  const int toff = seq_tile_offset(p.cu, b);
  // q of the group's heads as fp32 channel pairs q2[pair][g] (tail path and fragments)
  for (int x = t; x < (D / 2) * GRP; x += kDecThreads) {
    const int cp = x / GRP, gq = x % GRP;
    float2 v = make_float2(0.0f, 0.0f);
    if (gq < grp) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(
          p.q + ((long long)b * p.Hq + kvh * grp + gq) * D + 2 * cp);
      v = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    }
    q2[cp * GRP + gq] = v;
  }
  __syncthreads();
  // q of head h as a fixed-point integer Q of NL int8 limbs (balanced base-256
  // digits) times the power of two 2^(E_h - F), where 2^E_h > max_c |q_h[c]|:
  //   NL = 2, F = 14:   Q = 256 hi + lo, |Q| <= 2^14; a channel is off by at most
  //                    2^(E_h - 15) (exact within 2^7 of the head's largest |q|);
  //   NL = 3, F = 22:   Q = 65536 hi + 256 mid + lo, |Q| <= 2^22, off by at most
  //                    2^(E_h - 23) (exact within 2^15 of the largest |q|).
  // The error of two limbs grows with |q| in absolute terms, so they serve only groups
  // whose heads all have max |q| < 2^kTwoLimbMaxE.  Every step launches the kernel for
  // both limb counts; each (sequence, KV head) group takes part in exactly one of them,
  // and a CTA of the other leaves here, before it touches the tail or any counter.
  int* const qe = reinterpret_cast<int*>(sm + C::kOffE);
  for (int hd = warp; hd < GRP; hd += kConsumers + 1) {
    float mx = 0.0f;
    for (int cp = lane; cp < D / 2; cp += 32) {
      const float2 v = q2[cp * GRP + hd];
      mx = fmaxf(mx, fmaxf(fabsf(v.x), fabsf(v.y)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    int e = 0;
    frexpf(mx, &e);  // mx = f 2^e with f in [0.5, 1), or e = 0 for mx = 0
    if (lane == 0) qe[hd] = e;
  }
  __syncthreads();
  {
    bool three = false;
    for (int hd = 0; hd < grp; ++hd) three |= qe[hd] > kTwoLimbMaxE;
    if (three != (NL == 3)) return;  // uniform over the CTA
  }
  constexpr int F = NL == 3 ? 22 : 14;             // fraction bits of Q
  constexpr int QL = NL == 3 ? C::kQM + 1 : C::kQM;  // score MMAs per K fragment
  const int tl = __ldg(p.tail_len + b);
  if (tl >= p.tail_cap) {  // every CTA of sequence b leaves: output and tail untouched
    if (tail_cta && kvh == 0 && t == 0) atomicOr(p.status, TRA_DEV_TAIL_FULL);
    return;
  }
  int my0 = 0, ntile = 0;
  {
    // cached tiles of (b, kvh): the decode-cache list row, or (hybrid) every prefix
    // tile in INT4, my0 then being the split's first k-tile
    int rs = 0, n = (T + kTile - 1) / kTile;
    if (!HYB) {
      const long long row = (long long)b * p.Hkv + kvh;
      rs = __ldg(p.row_ptr + row);
      n = __ldg(p.row_ptr + row + 1) - rs;
    }
    my0 = rs + (int)((long long)n * split / nsplit);
    ntile = rs + (int)((long long)n * (split + 1) / nsplit) - my0;
  }
  // entry i of this split: (precision << 28) | kt
  auto entry_of = [&](int i) -> uint32_t {
    return HYB ? ((uint32_t)TRA_PREC_INT4 << 28) | (uint32_t)(my0 + i) : __ldg(p.entries + my0 + i);
  };
  // barriers first, so that the producer's first copies overlap the consumers' set-up
  if (t == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(bar_full + s * 8, 1);
      mbar_init(bar_empty + s * 8, 1);
    }
    *err = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < ntile; ++i) {
        const int s = i % kDecStages, use = i / kDecStages;
        if (use > 0 && !mbar_wait(bar_empty + s * 8, (use - 1) & 1, err)) break;
        const uint32_t e = entry_of(i);
        const int kt = (int)(e & 0x0FFFFFFFu);
        const int r0 = (kvh * p.ntiles + toff + kt) * kTile;
        const uint32_t dst = base + s * C::kStageBytes;
        if ((e >> 28) == TRA_PREC_INT8) {
          mbar_arrive_expect_tx(bar_full + s * 8, 2 * kTile * C::kRow8);
          tma_load_2d(dst, &m.k8, bar_full + s * 8, 0, r0);
          tma_load_2d(dst + C::kTileBytes, &m.v8, bar_full + s * 8, 0, r0);
        } else {
          mbar_arrive_expect_tx(bar_full + s * 8, 2 * kTile * C::kRow4);
          tma_load_2d(dst, &m.k4, bar_full + s * 8, 0, r0);
          tma_load_2d(dst + C::kTileBytes, &m.v4, bar_full + s * 8, 0, r0);
        }
        ++issued;
      }
      if (*err) {
        // an abandoned split: every load issued lands before the CTA can exit (this
        // thread alone arrives on the full barriers, so the last fill of each stage
        // completes its phase as soon as its bytes are in)
        for (int s = 0; s < kDecStages && s < issued; ++s)
          mbar_wait_drain(bar_full + s * 8, (uint32_t)(((issued - 1 - s) / kDecStages) & 1));
      }
    }
    named_sync(1);  // ring drained
    named_sync(2);  // merge area written
  } else {
    // ------------------------------------------------------------ consumers
    // append the new token to the tail (tail split; the tail slot tl is read by nobody)
    if (tail_cta) {
      const long long src = ((long long)b * p.Hkv + kvh) * D;
      const long long dst = (((long long)b * p.Hkv + kvh) * p.tail_cap + tl) * D;
      for (int c = t; c < D; c += 32 * kConsumers) {
        p.k_tail[dst + c] = p.k_new[src + c];
        p.v_tail[dst + c] = p.v_new[src + c];
      }
    }
    // zero the P rows of padded heads (never written; N = 8 heads per MMA)
    {
      __half* pz = reinterpret_cast<__half*>(sm + C::kOffP);
      for (int x = t; x < kConsumers * 8 * C::kPStride; x += 32 * kConsumers) pz[x] = __float2half(0.0f);
    }
    asm volatile("bar.sync 3, %0;" ::"n"(32 * kConsumers) : "memory");  // consumers only
    const int g = lane >> 2, tq = lane & 3;  // fragment group / thread in group
    bool real[C::kQM];
#pragma unroll
    for (int mq = 0; mq < C::kQM; ++mq) real[mq] = tq + 4 * mq < grp;
    // softmax state per slot (l_run: this lane's partial sum over its keys, reduced
    // over the lanes once at the end); O^T fragments o8[j]: channels 16j + 2g (rows g) and
    // 16j + 2g + 1 (rows g + 8), for INT8 and INT4 tiles alike (the V4 cache is stored
    // in this fragment order)
    float m_run[C::kQM], l_run[C::kQM];
#pragma unroll
    for (int mq = 0; mq < C::kQM; ++mq) {
      m_run[mq] = -INFINITY;
      l_run[mq] = 0.0f;
    }
    float o8[C::kB8][4];
#pragma unroll
    for (int j = 0; j < C::kB8; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) o8[j][k] = 0.0f;
    __half* const pw = reinterpret_cast<__half*>(sm + C::kOffP) + warp * 8 * C::kPStride;
    const uint32_t pw_addr = smem_u32(pw);
    const int mrow = lane & 7, mj = lane >> 3;  // ldmatrix: this lane's row / matrix
    // ldmatrix addresses: this lane's row of key block k is 16k + mrow + 8 (mj & 1),
    // its 16-byte chunk 2 cb + (mj >> 1).  Key blocks are 8-row aligned, so the TMA
    // swizzle term of the row is the same for every k: per-lane offsets per channel
    // block, plus 16 k rows.
    uint32_t off8[D / 32], off4[D / 64];
#pragma unroll
    for (int cb = 0; cb < D / 32; ++cb)
      off8[cb] = swz<C::kRow8>(mrow + 8 * (mj & 1), 2 * cb + (mj >> 1));
#pragma unroll
    for (int cb = 0; cb < D / 64; ++cb)
      off4[cb] = swz<C::kRow4>(mrow + 8 * (mj & 1), 2 * cb + (mj >> 1));

    // bf16 rows: the tail (tail CTA: tokens [0, tl) of the tail buffer and the new
    // token at tl) and, for the hybrid, the split's share of the selected and in-window
    // prefix rows.  row(x, kr, vr) gives row x's K and V and whether it takes part.
    // Warp w takes rows w, w + kConsumers, ..., one per lane, with CUDA-core fp32 math
    // and its own softmax state.  All of a lane's loads are issued before use.
    auto row_pass = [&](int count, auto row, float (&tm)[GRP], float (&tlsum)[GRP],
                        float2 (&to)[GRP][C::kCh / 2]) {
      for (int c0 = 0; warp + kConsumers * c0 < count; c0 += 32) {  // this warp's next 32 rows
        const int x = warp + kConsumers * (c0 + lane);
        const uint16_t* kr = nullptr;
        const uint16_t* vr0 = nullptr;
        const bool valid = x < count && row(x, kr, vr0);
        float2 acc[GRP];
#pragma unroll
        for (int gg = 0; gg < GRP; ++gg) acc[gg] = make_float2(0.0f, 0.0f);
        if (valid) {
          uint4 kw[D / 8];
#pragma unroll
          for (int c = 0; c < D / 8; ++c) kw[c] = *reinterpret_cast<const uint4*>(kr + c * 8);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            const uint32_t ww[4] = {kw[c].x, kw[c].y, kw[c].z, kw[c].w};
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const float2 kk = make_float2(__uint_as_float(ww[x] << 16),
                                            __uint_as_float(ww[x] & 0xFFFF0000u));
#pragma unroll
              for (int gg = 0; gg < GRP; ++gg)
                acc[gg] = __ffma2_rn(kk, q2[(c * 4 + x) * GRP + gg], acc[gg]);
            }
          }
        }
        float pk[GRP], al[GRP];
#pragma unroll
        for (int gg = 0; gg < GRP; ++gg) {
          const float sc = valid ? (acc[gg].x + acc[gg].y) * p.scale_log2 : -INFINITY;
          float mx = sc;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const float m_new = fmaxf(tm[gg], mx);
          const float mb = m_new == -INFINITY ? 0.0f : m_new;
          pk[gg] = valid ? ex2(sc - mb) : 0.0f;
          float ps = pk[gg];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
          al[gg] = ex2(tm[gg] - mb);  // -inf -> 0
          tlsum[gg] = tlsum[gg] * al[gg] + ps;
          tm[gg] = m_new;
        }
#pragma unroll
        for (int gg = 0; gg < GRP; ++gg)
#pragma unroll
          for (int k = 0; k < C::kCh / 2; ++k)
            to[gg][k] = __fmul2_rn(to[gg][k], make_float2(al[gg], al[gg]));
        // P V: this lane's channels lane * kCh .. + kCh, rows of the chunk in order
        const int nk = min(32, (count - 1 - warp) / kConsumers - c0 + 1);
#pragma unroll 4
        for (int j = 0; j < nk; ++j) {
          const int pj = warp + kConsumers * (c0 + j);
          const uint16_t* kr_unused = nullptr;
          const uint16_t* vr = nullptr;
          if (!row(pj, kr_unused, vr)) continue;  // (uniform over the warp)
          uint32_t vw[C::kCh / 2];
#pragma unroll
          for (int k = 0; k < C::kCh / 2; ++k)
            vw[k] = *reinterpret_cast<const uint32_t*>(vr + lane * C::kCh + 2 * k);
#pragma unroll
          for (int gg = 0; gg < GRP; ++gg) {
            const float pv = __shfl_sync(0xffffffffu, pk[gg], j);
#pragma unroll
            for (int k = 0; k < C::kCh / 2; ++k)
              to[gg][k] = __ffma2_rn(make_float2(__uint_as_float(vw[k] << 16),
                                                 __uint_as_float(vw[k] & 0xFFFF0000u)),
                                     make_float2(pv, pv), to[gg][k]);
          }
        }
      }
    };

    bool ok = true;
    // limb `limb` of head hd's Q at channel c (two limbs: 0 hi, 1 lo; three: 0 hi,
    // 1 mid, 2 lo; each in [-128, 127]); 0 for padded heads
    auto q_limb = [&](int hd, int limb, int c) -> uint32_t {
      if (hd >= grp) return 0u;
      const float2 v = q2[(c >> 1) * GRP + hd];
      const int Q = __float2int_rn(ldexpf(c & 1 ? v.y : v.x, F - qe[hd]));
      const int lo = ((Q + 128) & 0xFF) - 128;
      const int q1 = (Q - lo) >> 8;
      if (NL == 2) return (uint32_t)((limb == 0 ? q1 : lo) & 0xFF);
      const int mid = ((q1 + 128) & 0xFF) - 128;
      const int hi = (q1 - mid) >> 8;
      return (uint32_t)((limb == 0 ? hi : limb == 1 ? mid : lo) & 0xFF);
    };
    auto pack4 = [&](int hd, int limb, int c, int step) -> uint32_t {
      return q_limb(hd, limb, c) | q_limb(hd, limb, c + step) << 8 |
             q_limb(hd, limb, c + 2 * step) << 16 | q_limb(hd, limb, c + 3 * step) << 24;
    };
    // B fragments.  MMA mq < kQM: column g = (head (g >> 1) + 4 mq, limb g & 1), so
    // lane tq's accumulator columns 2tq, 2tq + 1 are the first two limb products (hi,
    // lo for two limbs; hi, mid for three) of head tq + 4 mq.  With three limbs, MMA
    // kQM: column g = lo limb of head (g >> 1) + 4 (g & 1), so lane tq's columns hold
    // the lo products of heads tq and tq + 4.
    // Channel order as the K codes arrive:
    //   INT8, 32-channel block cb: k = 4t + i -> channel 32cb + 4t + i, k = 16 + 4t + i
    //         -> 32cb + 16 + 4t + i
    //   INT4, 32-channel block 2cb + h: k = 4t + i -> even channel 64cb + 32h + 8t + 2i,
    //         k = 16 + 4t + i -> the odd channel after it
    uint32_t qi8[D / 32][QL][2], qi4[D / 64][2][QL][2];
  #pragma unroll
    for (int mq = 0; mq < QL; ++mq) {
      const bool lo_mma = NL == 3 && mq == C::kQM;
      const int hc = lo_mma ? (g >> 1) + 4 * (g & 1) : (g >> 1) + 4 * mq;
      const int limb = lo_mma ? 2 : (g & 1);
  #pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        qi8[cb][mq][0] = pack4(hc, limb, 32 * cb + 4 * tq, 1);
        qi8[cb][mq][1] = pack4(hc, limb, 32 * cb + 16 + 4 * tq, 1);
      }
  #pragma unroll
      for (int cb = 0; cb < D / 64; ++cb)
  #pragma unroll
        for (int h = 0; h < 2; ++h) {
          qi4[cb][h][mq][0] = pack4(hc, limb, 64 * cb + 32 * h + 8 * tq, 2);
          qi4[cb][h][mq][1] = pack4(hc, limb, 64 * cb + 32 * h + 8 * tq + 1, 2);
        }
    }
    float qsig[C::kQM];  // 2^(E - F) of the lane's softmax heads tq + 4 mq
#pragma unroll
    for (int mq = 0; mq < C::kQM; ++mq)
      qsig[mq] = real[mq] ? ldexpf(1.0f, qe[tq + 4 * mq] - F) : 0.0f;
    // hybrid: the selected-key mask of this warp's next tile, loaded a tile ahead
    uint64_t hi_next = (HYB && warp < ntile)
                           ? __ldg(p.sel_mask + (long long)kvh * p.ntiles + toff + my0 + warp) : 0ull;
    for (int i = warp; i < ntile; i += kConsumers) {
      const int s = i % kDecStages;
      const uint64_t hi_sel = hi_next;
      if (HYB && i + kConsumers < ntile)
        hi_next = __ldg(p.sel_mask + (long long)kvh * p.ntiles + toff + my0 + i + kConsumers);
      // Stage s last held tile i - kDecStages, which another warp consumes.  A
      // parity wait only tells adjacent phases apart, so this warp first waits for
      // that tile's release (which the load of tile i needs anyway): only then is the
      // full barrier's previous phase known to be complete, and its wait exact.  The
      // release wait is itself exact: the tile before that one in stage s was released
      // before tile i - kDecStages was loaded, which happened no later than this
      // warp's previous tile i - kConsumers (kConsumers <= kDecStages).
      if (i >= kDecStages &&
          !mbar_wait(bar_empty + s * 8, ((i / kDecStages) - 1) & 1, err)) { ok = false; break; }
      if (!mbar_wait(bar_full + s * 8, (i / kDecStages) & 1, err)) { ok = false; break; }
      const uint32_t e = entry_of(i);
      const int kt = (int)(e & 0x0FFFFFFFu);
      const long long tile = (long long)kvh * p.ntiles + toff + kt;
      const int nvalid = min(kTile, T - kt * kTile);
      const uint32_t kb = base + s * C::kStageBytes;
      const uint32_t vb = kb + C::kTileBytes;
      const bool is8 = (e >> 28) == TRA_PREC_INT8;

      // ---- scores: si[mq][k] = S^T fragment of keys 16k + (g, g+8), columns (2tq, 2tq+1)
      int si[QL][4][4];
  #pragma unroll
      for (int mq = 0; mq < QL; ++mq)
  #pragma unroll
        for (int k = 0; k < 4; ++k)
  #pragma unroll
          for (int x = 0; x < 4; ++x) si[mq][k][x] = 0;
      if (is8) {
  #pragma unroll
        for (int cb = 0; cb < D / 32; ++cb)
  #pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t r[4];  // keys g / g+8 at channels 32cb + 4tq .. (+16): the A fragment as is
            ldsm_x4(kb + 16 * C::kRow8 * k + off8[cb], r);
  #pragma unroll
            for (int mq = 0; mq < QL; ++mq) mma_s8(si[mq][k], r, qi8[cb][mq][0], qi8[cb][mq][1]);
          }
      } else {
  #pragma unroll
        for (int cb = 0; cb < D / 64; ++cb)
  #pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t r[4];
            ldsm_x4(kb + 16 * C::kRow4 * k + off4[cb], r);
  #pragma unroll
            for (int h = 0; h < 2; ++h) {  // packed bytes 16h.. = channels 64cb + 32h ..
              // keys g / g+8, channels 8tq + (0, 2, 4, 6) and 8tq + (1, 3, 5, 7)
              const uint32_t a[4] = {i4_even_x16(r[2 * h]), i4_even_x16(r[2 * h + 1]),
                                     i4_odd_x16(r[2 * h]), i4_odd_x16(r[2 * h + 1])};
  #pragma unroll
              for (int mq = 0; mq < QL; ++mq)
                mma_s8(si[mq][k], a, qi4[cb][h][mq][0], qi4[cb][h][mq][1]);
            }
          }
      }
      // ---- online softmax for this lane's slots over keys 16k + g (+8): accumulator
      // columns 2tq, 2tq + 1 of MMA mq hold the hi and mid limb products of head
      // tq + 4 mq, column 2tq + mq of MMA kQM its lo limb products
      const float kscale = (is8 ? __ldg(p.sk8 + tile) : __ldg(p.sk4 + tile) * 0.0625f) * p.scale_log2;
      const float vs = is8 ? __ldg(p.sv8 + tile) : __ldg(p.sv4 + tile);
      float sv[C::kQM][8];  // [slot][key slot: 2k + (g / g+8)]
  #pragma unroll
      for (int mq = 0; mq < C::kQM; ++mq) {
        const float ks = kscale * qsig[mq];
  #pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (NL == 2) {
            sv[mq][2 * k] = (float)(si[mq][k][0] * 256 + si[mq][k][1]) * ks;
            sv[mq][2 * k + 1] = (float)(si[mq][k][2] * 256 + si[mq][k][3]) * ks;
          } else {
            // hi x 65536 is exact in fp32 (|hi| < 2^21); mid x 256 + lo fits int32
            sv[mq][2 * k] = fmaf((float)si[mq][k][0], 65536.0f,
                                 (float)(si[mq][k][1] * 256 + si[QL - 1][k][mq])) * ks;
            sv[mq][2 * k + 1] = fmaf((float)si[mq][k][2], 65536.0f,
                                     (float)(si[mq][k][3] * 256 + si[QL - 1][k][2 + mq])) * ks;
          }
        }
      }
      if (HYB) {
        // selected keys and keys within the window of the query (position T + tl) are
        // read in bf16 by the row pass: masked out of their INT4 tile here
        uint64_t hi = hi_sel;
        const int wlo = T + tl - p.window + 1 - kt * kTile;  // first in-window key of the tile
        if (p.window > 0 && wlo < kTile) hi |= wlo <= 0 ? ~0ull : (~0ull << wlo);
        if (hi) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int mq = 0; mq < C::kQM; ++mq) {
              if ((hi >> (16 * k + g)) & 1) sv[mq][2 * k] = -INFINITY;
              if ((hi >> (16 * k + g + 8)) & 1) sv[mq][2 * k + 1] = -INFINITY;
            }
        }
      }
      if (nvalid < kTile) {  // a sequence's last tile: keys past its end are masked
  #pragma unroll
        for (int k = 0; k < 4; ++k)
  #pragma unroll
          for (int mq = 0; mq < C::kQM; ++mq) {
            if (16 * k + g >= nvalid) sv[mq][2 * k] = -INFINITY;
            if (16 * k + g + 8 >= nvalid) sv[mq][2 * k + 1] = -INFINITY;
          }
      }
      float mt[C::kQM], alpha[C::kQM];
      bool need = false;
  #pragma unroll
      for (int mq = 0; mq < C::kQM; ++mq) {
        float x = sv[mq][0];
  #pragma unroll
        for (int k = 1; k < 8; ++k) x = fmaxf(x, sv[mq][k]);
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
        mt[mq] = x;
        alpha[mq] = 1.0f;
        need |= fmaxf(m_run[mq], x) > m_run[mq] + 8.0f;  // true for the first finite max
      }
      // lazy rescaling: the reference max moves only when it grew by more than 2^8
      const bool warp_need = __any_sync(0xffffffffu, need);
      if (warp_need) {
  #pragma unroll
        for (int mq = 0; mq < C::kQM; ++mq) {
          const float m_new = fmaxf(m_run[mq], mt[mq]);
          if (m_new > m_run[mq]) {
            alpha[mq] = ex2(m_run[mq] - m_new);  // -inf -> 0
            m_run[mq] = m_new;
          }
        }
      }
  #pragma unroll
      for (int mq = 0; mq < C::kQM; ++mq) {
        const float mb = m_run[mq] == -INFINITY ? 0.0f : m_run[mq];
        float ps = 0.0f;
        __half* prow = pw + (tq + 4 * mq) * C::kPStride;
  #pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float p0 = real[mq] ? ex2(sv[mq][2 * k] - mb) : 0.0f;
          const float p1 = real[mq] ? ex2(sv[mq][2 * k + 1] - mb) : 0.0f;
          ps += p0 + p1;
          prow[16 * k + g] = __float2half_rn(p0 * vs);
          prow[16 * k + g + 8] = __float2half_rn(p1 * vs);
        }
        l_run[mq] = l_run[mq] * alpha[mq] + ps;
      }
      if (warp_need) {
        // O head 2tq + hh is softmax slot (2tq + hh) / 4 of lane 4g + (2tq + hh) % 4
        float ao[2];
  #pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int hd = 2 * tq + hh, src = (lane & ~3) | (hd & 3);
          const float a0 = __shfl_sync(0xffffffffu, alpha[0], src);
          const float a1 = __shfl_sync(0xffffffffu, alpha[C::kQM - 1], src);
          ao[hh] = hd >= 4 ? a1 : a0;
        }
  #pragma unroll
        for (int j = 0; j < C::kB8; ++j) {
          o8[j][0] *= ao[0]; o8[j][1] *= ao[1];
          o8[j][2] *= ao[0]; o8[j][3] *= ao[1];
        }
      }
      __syncwarp();
      // ---- O^T += V^T P^T: B fragment = P[head g][keys 16k + 2tq (+1), +8 (+9)]
  #pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t pb0, pb1;
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(pb0) : "r"(pw_addr + (g * C::kPStride + 16 * k + 2 * tq) * 2));
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(pb1) : "r"(pw_addr + (g * C::kPStride + 16 * k + 2 * tq + 8) * 2));
        if (is8) {
  #pragma unroll
          for (int cp = 0; cp < D / 32; ++cp) {
            uint32_t r[4];
            ldsm_x4_t(vb + 16 * C::kRow8 * k + off8[cp], r);
  #pragma unroll
            for (int h = 0; h < 2; ++h) {  // channels 32cp + 16h + (2g, 2g+1)
              // V8 codes are stored offset-binary (code + 128)
              const uint32_t u0 = r[2 * h], u1 = r[2 * h + 1];
              const uint32_t a[4] = {h2_from_bytes(u0, kSel02, kBias8), h2_from_bytes(u0, kSel13, kBias8),
                                     h2_from_bytes(u1, kSel02, kBias8), h2_from_bytes(u1, kSel13, kBias8)};
              mma16816(o8[2 * cp + h], a, pb0, pb1);
            }
          }
        } else {
  #pragma unroll
          for (int cp = 0; cp < D / 64; ++cp) {
            uint32_t r[4];
            ldsm_x4_t(vb + 16 * C::kRow4 * k + off4[cp], r);
  #pragma unroll
            for (int h = 0; h < 2; ++h) {  // 32 channels 64cp + 32h ..
              // words: keys (2tq, 2tq+1) / (2tq+8, 2tq+9); nibble n of the lane's 16-bit
              // column holds channel 64cp + 32h + 16 (n / 2) + 2g + n % 2, so the
              // conversion yields one key pair per channel of blocks 4cp + 2h (+1)
              uint32_t v0[4], v1[4];
              i4x8_to_h2(r[2 * h], v0);
              i4x8_to_h2(r[2 * h + 1], v1);
              const uint32_t aA[4] = {v0[0], v0[1], v1[0], v1[1]};
              mma16816(o8[4 * cp + 2 * h], aA, pb0, pb1);
              const uint32_t aB[4] = {v0[2], v0[3], v1[2], v1[3]};
              mma16816(o8[4 * cp + 2 * h + 1], aB, pb0, pb1);
            }
          }
        }
      }
      // stage s and this warp's P rows may be reused once every lane is done
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + s * 8);
    }

    // ---- the shared-memory merge; the merge area aliases the ring, so every warp
    // must be done with the ring first.  Slot w holds warp w's tile state, slot
    // kConsumers + w (the tail split only) its tail state.
    float* rw = red + warp * GRP * (D + 2);
#pragma unroll
    for (int mq = 0; mq < C::kQM; ++mq)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) l_run[mq] += __shfl_xor_sync(0xffffffffu, l_run[mq], o);
    named_sync(1);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int hd = 2 * tq + hh;
      if (hd < GRP) {
#pragma unroll
        for (int j = 0; j < C::kB8; ++j) {
          rw[hd * (D + 2) + 16 * j + 2 * g] = o8[j][hh];
          rw[hd * (D + 2) + 16 * j + 2 * g + 1] = o8[j][2 + hh];
        }
      }
    }
#pragma unroll
    for (int mq = 0; mq < C::kQM; ++mq) {
      const int hd = tq + 4 * mq;
      if (hd < GRP && g == 0) {
        rw[hd * (D + 2) + D] = m_run[mq];
        rw[hd * (D + 2) + D + 1] = l_run[mq];
      }
    }
    if (HYB || tail_cta) {
      float tm[GRP], tlsum[GRP];
      float2 to[GRP][C::kCh / 2];
#pragma unroll
      for (int gg = 0; gg < GRP; ++gg) {
        tm[gg] = -INFINITY;
        tlsum[gg] = 0.0f;
#pragma unroll
        for (int k = 0; k < C::kCh / 2; ++k) to[gg][k] = make_float2(0.0f, 0.0f);
      }
      const long long tbase = ((long long)b * p.Hkv + kvh) * p.tail_cap;
      const long long nbase = ((long long)b * p.Hkv + kvh) * D;
      auto tail_row = [&](int x, const uint16_t*& kr, const uint16_t*& vr) -> bool {
        kr = x == tl ? p.k_new + nbase : p.k_tail + (tbase + x) * D;
        vr = x == tl ? p.v_new + nbase : p.v_tail + (tbase + x) * D;
        return true;
      };
      const int ntail = tail_cta ? tl + 1 : 0;
      if (!HYB) {
        row_pass(ntail, tail_row, tm, tlsum, to);
      } else {
        // hybrid bf16 rows: n_sel selected rows, then `window` rows of the last prefix
        // tokens (a window row takes part if it is still in the query's window and not
        // selected); split x takes rows [R x / S, R (x + 1) / S) of the R, then the tail
        const int nsel = __ldg(p.sel_count + b);
        const int R = nsel + p.window;
        const int x0 = (int)((long long)R * split / nsplit);
        const int nh = (int)((long long)R * (split + 1) / nsplit) - x0;
        const long long sbase = ((long long)b * p.Hkv + kvh) * p.sel_cap;
        const long long wbase = ((long long)b * p.Hkv + kvh) * p.window;
        const int qpos = T + tl;  // the query's position
        auto hy_row = [&](int x, const uint16_t*& kr, const uint16_t*& vr) -> bool {
          if (x >= nh) return tail_row(x - nh, kr, vr);
          const int hx = x0 + x;
          if (hx < nsel) {
            kr = p.k_sel + (sbase + hx) * D;
            vr = p.v_sel + (sbase + hx) * D;
            return true;
          }
          const int w = hx - nsel, j = T - p.window + w;
          kr = p.k_win + (wbase + w) * D;
          vr = p.v_win + (wbase + w) * D;
          if (j < 0 || qpos - j >= p.window) return false;
          const uint64_t sm_ = __ldg(p.sel_mask + (long long)kvh * p.ntiles + toff + j / kTile);
          return ((sm_ >> (j % kTile)) & 1) == 0;
        };
        row_pass(nh + ntail, hy_row, tm, tlsum, to);
      }
      float* rt = red + (kConsumers + warp) * GRP * (D + 2);
#pragma unroll
      for (int gg = 0; gg < GRP; ++gg) {
#pragma unroll
        for (int k = 0; k < C::kCh / 2; ++k)
          *reinterpret_cast<float2*>(rt + gg * (D + 2) + lane * C::kCh + 2 * k) = to[gg][k];
        if (lane == 0) {
          rt[gg * (D + 2) + D] = tm[gg];
          rt[gg * (D + 2) + D + 1] = tlsum[gg];
        }
      }
    }
    named_sync(2);
  }
  // merge the consumer warps' states into this split's partial (m, l, o)
  const int nstates = (HYB || tail_cta) ? C::kStates : kConsumers;
  for (int x = t; x < GRP * D; x += kDecThreads) {
    const int gg = x / D, c = x % D;
    if (gg >= grp) continue;
    float M = -INFINITY;
    for (int w = 0; w < nstates; ++w) M = fmaxf(M, red[(w * GRP + gg) * (D + 2) + D]);
    float L = 0.0f, o = 0.0f;
    for (int w = 0; w < nstates; ++w) {
      const float* r = red + (w * GRP + gg) * (D + 2);
      const float wt = r[D] == -INFINITY ? 0.0f : ex2(r[D] - M);
      L += r[D + 1] * wt;
      o += r[c] * wt;
    }
    const long long pi = ((long long)b * p.Hq + kvh * grp + gg) * p.splits + blockIdx.x;
    p.part_o[pi * D + c] = o;
    if (c == 0) {
      p.part_ml[pi * 2] = M;
      p.part_ml[pi * 2 + 1] = L;
    }
  }
  if (t == 0 && *err) atomicOr(p.status, *err);

  // The last split of row (b, kvh) to finish merges the row's partials into the
  // output of its query heads (a release / acquire pair of fences around the
  // arrival count); the last row of sequence b advances tail_len[b], which every
  // CTA of the sequence has read by then.
  volatile int* const last = err + 1;
  const long long row = (long long)b * p.Hkv + kvh;
  __threadfence();
  __syncthreads();
  if (t == 0) *last = atomicAdd(p.row_count + row, 1) == p.splits - 1;
  __syncthreads();
  if (!*last) return;
  __threadfence();
  // (m, l) of the row's (head, split) partials into shared memory (the ring is
  // free), then per head the max M, the weights 2^(m - M) and 1/L, then O
  const int S = p.splits;
  const long long hb = (long long)b * p.Hq + kvh * grp;  // first query head of the row
  float* const wm = reinterpret_cast<float*>(sm);        // [grp][S] m, then weights
  float* const wl = wm + GRP * TRA_MAX_DECODE_SPLITS;    // [grp][S] l
  float* const winv = wl + GRP * TRA_MAX_DECODE_SPLITS;  // [grp] 1 / L
  for (int x = t; x < grp * S; x += kDecThreads) {
    wm[x] = __ldcg(p.part_ml + (hb * S + x) * 2);
    wl[x] = __ldcg(p.part_ml + (hb * S + x) * 2 + 1);
  }
  __syncthreads();
  if (t < grp) {
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, wm[t * S + s]);
    float L = 0.0f;
    for (int s = 0; s < S; ++s) {
      const float m = wm[t * S + s];
      const float wt = m == -INFINITY ? 0.0f : ex2(m - M);
      wm[t * S + s] = wt;
      L += wl[t * S + s] * wt;
    }
    winv[t] = L > 0.0f ? 1.0f / L : 0.0f;
  }
  __syncthreads();
  for (int x = t; x < grp * D; x += kDecThreads) {
    const int gg = x / D, c = x % D;
    const float* po = p.part_o + (hb + gg) * S * D + c;
    float o = 0.0f;
#pragma unroll 4
    for (int s = 0; s < S; ++s) o += __ldcg(po + (long long)s * D) * wm[gg * S + s];
    const __nv_bfloat16 r = __float2bfloat16_rn(o * winv[gg]);
    p.out[(hb + gg) * D + c] = *reinterpret_cast<const uint16_t*>(&r);
  }
  if (t == 0) {
    p.row_count[row] = 0;
    __threadfence();
    if (atomicAdd(p.seq_count + b, 1) == p.Hkv - 1) {
      p.seq_count[b] = 0;
      p.tail_len[b] += 1;
    }
  }
}

template <int D, int GRP, bool HYB>
cudaError_t launch_dec_h(const DecodeParams& p, const DecodeMaps& m, cudaStream_t s) {
  using C = DecCfg<D, GRP>;
  dim3 grid(p.splits, p.Hkv, p.B);
  // two limbs first (the common case), then three; each group runs in one of them
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, GRP, 2, HYB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  decode_split_kernel<D, GRP, 2, HYB><<<grid, kDecThreads, C::kSmem, s>>>(p, m);
  e = cudaFuncSetAttribute(decode_split_kernel<D, GRP, 3, HYB>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  decode_split_kernel<D, GRP, 3, HYB><<<grid, kDecThreads, C::kSmem, s>>>(p, m);
  return cudaGetLastError();
}

template <int D, int GRP>
cudaError_t launch_dec(const DecodeParams& p, const DecodeMaps& m, cudaStream_t s) {
  return p.sel_mask ? launch_dec_h<D, GRP, true>(p, m, s) : launch_dec_h<D, GRP, false>(p, m, s);
}

template <int D>
cudaError_t launch_dec_d(const DecodeParams& p, const DecodeMaps& m, cudaStream_t s) {
  const int grp = p.Hq / p.Hkv;
  if (grp <= 1) return launch_dec<D, 1>(p, m, s);
  if (grp <= 2) return launch_dec<D, 2>(p, m, s);
  if (grp <= 4) return launch_dec<D, 4>(p, m, s);
  return launch_dec<D, 8>(p, m, s);
}

}  // namespace

// Splits (partials) per (sequence, KV head); the last one also takes the tail.
int decode_splits(int B, int Hkv) {
  // about 256 CTAs: long CTAs, little set-up and a short merge, one wave of two CTAs
  // per SM at batch 16 x 8 KV heads
  const int target = 256;
  const int rows = B * Hkv;
  int s = (target + rows - 1) / rows;
  if (s < 1) s = 1;
  if (s > TRA_MAX_DECODE_SPLITS) s = TRA_MAX_DECODE_SPLITS;
  return s;
}

cudaError_t launch_decode(const DecodeParams& p, const DecodeMaps& m, cudaStream_t s) {
  return p.d == 128 ? launch_dec_d<128>(p, m, s) : launch_dec_d<64>(p, m, s);
}

}  // namespace tra
