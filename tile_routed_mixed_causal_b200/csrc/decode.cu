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
//   scores: lane j owns keys j and j+32; codes become exact floats (byte
//           permute into the mantissa of 2^23, then one packed subtraction) and
//           meet q (fp32, broadcast from shared memory) in packed fp32x2 FMAs;
//   softmax: warp max / sum per head, K scale and 1/sqrt(d) folded into the
//           exponent, V scale folded into P;
//   P V:    lane l owns D/32 consecutive channels and accumulates o for every head.
// The last split also covers the bf16 tail (earlier decode tokens + the new
// one).  The four warps' states are merged per CTA, and a small combine kernel
// merges the splits and advances tail_len.
#include "tra_device.cuh"
#include "tra_launch.h"

namespace tra {
namespace {

constexpr int kConsumers = 4;
constexpr int kDecThreads = 32 * (kConsumers + 1);
constexpr int kDecStages = 6;

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

// Four signed INT8 codes of a word -> two float2 (exact): each byte, offset by
// 128, is placed in the low mantissa byte of 2^23 and 2^23 + 128 is subtracted.
__device__ __forceinline__ void i8x4_to_f2(uint32_t w, float2& a, float2& b) {
  const uint32_t u = w ^ 0x80808080u;
  const float2 off = make_float2(-8388736.0f, -8388736.0f);
  a = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)),
                             __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651))),
                 off);
  b = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)),
                             __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653))),
                 off);
}

// Eight INT4 codes of a word (even channel in the low nibble) -> four float2.
__device__ __forceinline__ void i4x8_to_f2(uint32_t w, float2 (&f)[4]) {
  const uint2 e = expand_int4x8(w);  // eight int8 codes in channel order
  i8x4_to_f2(e.x, f[0], f[1]);
  i8x4_to_f2(e.y, f[2], f[3]);
}

template <int D, int GRP>
struct DecCfg {
  static constexpr int kRow8 = D;                // INT8 row bytes
  static constexpr int kRow4 = D / 2;            // INT4 row bytes
  static constexpr int kTileBytes = kTile * D;   // INT8 codes of one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kOffQ = kDecStages * kStageBytes;  // q: [D/2 pairs][GRP] float2
  static constexpr int kQBytes = (D / 2) * GRP * 8;
  static constexpr int kOffP = kOffQ + kQBytes;            // p: [warp][64 keys][GRP] float
  static constexpr int kPBytes = kConsumers * kTile * GRP * 4;
  static constexpr int kOffRed = kOffP + kPBytes;          // merge: [warp][GRP][D + 2] float
  static constexpr int kRedBytes = kConsumers * GRP * (D + 2) * 4;
  static constexpr int kOffBar = kOffRed + kRedBytes;
  static constexpr int kSmem = kOffBar + 2 * kDecStages * 8 + 16 + 1024;
  static constexpr int kCh = D / 32;             // P V channels per lane
};

template <int D, int GRP>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(
    const DecodeParams p, const __grid_constant__ DecodeMaps m) {
  using C = DecCfg<D, GRP>;
  extern __shared__ uint8_t dsm_raw[];
  const uint32_t base = (smem_u32(dsm_raw) + 1023u) & ~1023u;
  uint8_t* const sm = dsm_raw + (base - smem_u32(dsm_raw));
  float2* const q2 = reinterpret_cast<float2*>(sm + C::kOffQ);
  float* const p_sm = reinterpret_cast<float*>(sm + C::kOffP);
  float* const red = reinterpret_cast<float*>(sm + C::kOffRed);
  const uint32_t bar_full = base + C::kOffBar;
  const uint32_t bar_empty = bar_full + kDecStages * 8;
  volatile int* const err =
      reinterpret_cast<volatile int*>(sm + C::kOffBar + 2 * kDecStages * 8);

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int grp = p.Hq / p.Hkv;
  const int seq0 = __ldg(p.cu + b);
  const int T = __ldg(p.cu + b + 1) - seq0;
  const int toff = seq_tile_offset(p.cu, b);
  const int tl = __ldg(p.tail_len + b);
  if (tl >= p.tail_cap) {
    if (split == 0 && kvh == 0 && t == 0) {
      atomicOr(p.status, TRA_DEV_TAIL_FULL);
      p.skip[b] = 1;
    }
    return;
  }
  if (split == 0 && kvh == 0 && t == 0) p.skip[b] = 0;
  const long long row = (long long)b * p.Hkv + kvh;
  const int rs = __ldg(p.row_ptr + row), re = __ldg(p.row_ptr + row + 1);
  const int n = re - rs;
  const int my0 = rs + (int)((long long)n * split / p.splits);
  const int ntile = rs + (int)((long long)n * (split + 1) / p.splits) - my0;
  const bool last = split == p.splits - 1;

  // append the new token to the tail (split 0; the tail slot tl is read by nobody)
  if (split == 0) {
    const long long src = ((long long)b * p.Hkv + kvh) * D;
    const long long dst = (((long long)b * p.Hkv + kvh) * p.tail_cap + tl) * D;
    for (int c = t; c < D; c += kDecThreads) {
      p.k_tail[dst + c] = p.k_new[src + c];
      p.v_tail[dst + c] = p.v_new[src + c];
    }
  }
  // q of the group's heads as fp32 channel pairs: q2[pair][g]
  for (int x = t; x < (D / 2) * GRP; x += kDecThreads) {
    const int cp = x / GRP, g = x % GRP;
    float2 v = make_float2(0.0f, 0.0f);
    if (g < grp) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(
          p.q + ((long long)b * p.Hq + kvh * grp + g) * D + 2 * cp);
      v = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    }
    q2[cp * GRP + g] = v;
  }
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
      for (int i = 0; i < ntile; ++i) {
        const int s = i % kDecStages, use = i / kDecStages;
        if (use > 0 && !mbar_wait(bar_empty + s * 8, (use - 1) & 1, err)) break;
        const uint32_t e = __ldg(p.entries + my0 + i);
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
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    float m_run[GRP], l_run[GRP];
    float2 o2[GRP][C::kCh / 2];  // this lane's channels lane*kCh .. for every head
#pragma unroll
    for (int g = 0; g < GRP; ++g) {
      m_run[g] = -INFINITY;
      l_run[g] = 0.0f;
#pragma unroll
      for (int k = 0; k < C::kCh / 2; ++k) o2[g][k] = make_float2(0.0f, 0.0f);
    }
    float* const pw = p_sm + warp * kTile * GRP;

    // online-softmax update with this block's scores s[k][g] (lane keys j, j+32),
    // then P V with p * vscale staged in shared memory; vload(key, v) gives this
    // lane's channels of V row `key` as floats
    auto softmax_pv = [&](float (&s)[2][GRP], float vscale, auto vload) {
      float alpha[GRP];
#pragma unroll
      for (int g = 0; g < GRP; ++g) {
        float mt = fmaxf(s[0][g], s[1][g]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
        const float m_new = fmaxf(m_run[g], mt);
        const float mb = m_new == -INFINITY ? 0.0f : m_new;
        const float p0 = ex2(s[0][g] - mb), p1 = ex2(s[1][g] - mb);  // ex2(-inf) = 0
        float ps = p0 + p1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        alpha[g] = ex2(m_run[g] - mb);
        l_run[g] = l_run[g] * alpha[g] + ps;
        m_run[g] = m_new;
        pw[lane * GRP + g] = p0 * vscale;
        pw[(lane + 32) * GRP + g] = p1 * vscale;
      }
      __syncwarp();
#pragma unroll
      for (int g = 0; g < GRP; ++g)
#pragma unroll
        for (int k = 0; k < C::kCh / 2; ++k)
          o2[g][k] = __fmul2_rn(o2[g][k], make_float2(alpha[g], alpha[g]));
#pragma unroll 4
      for (int key = 0; key < kTile; ++key) {
        float2 v[C::kCh / 2];
        vload(key, v);
        float pp[GRP];
        if constexpr (GRP % 4 == 0) {
#pragma unroll
          for (int g = 0; g < GRP; g += 4) {
            const float4 q4 = *reinterpret_cast<const float4*>(pw + key * GRP + g);
            pp[g] = q4.x;
            pp[g + 1] = q4.y;
            pp[g + 2] = q4.z;
            pp[g + 3] = q4.w;
          }
        } else {
#pragma unroll
          for (int g = 0; g < GRP; ++g) pp[g] = pw[key * GRP + g];
        }
#pragma unroll
        for (int g = 0; g < GRP; ++g)
#pragma unroll
          for (int k = 0; k < C::kCh / 2; ++k)
            o2[g][k] = __ffma2_rn(v[k], make_float2(pp[g], pp[g]), o2[g][k]);
      }
      __syncwarp();
    };

    bool ok = true;
    for (int i = warp; i < ntile; i += kConsumers) {
      const int s = i % kDecStages;
      if (!mbar_wait(bar_full + s * 8, (i / kDecStages) & 1, err)) { ok = false; break; }
      const uint32_t e = __ldg(p.entries + my0 + i);
      const int kt = (int)(e & 0x0FFFFFFFu);
      const long long tile = (long long)kvh * p.ntiles + toff + kt;
      const int nvalid = min(kTile, T - kt * kTile);
      const uint8_t* kb = sm + s * C::kStageBytes;
      const uint8_t* vb = kb + C::kTileBytes;
      float sc[2][GRP];
      float2 acc[2][GRP];
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int g = 0; g < GRP; ++g) acc[k][g] = make_float2(0.0f, 0.0f);
      const bool is8 = (e >> 28) == TRA_PREC_INT8;
      if (is8) {
        // 16 codes (one swizzled chunk) per key per step
#pragma unroll 2
        for (int c = 0; c < C::kRow8 / 16; ++c) {
          const uint4 w0 = *reinterpret_cast<const uint4*>(kb + swz<C::kRow8>(lane, c));
          const uint4 w1 = *reinterpret_cast<const uint4*>(kb + swz<C::kRow8>(lane + 32, c));
          const uint32_t a0[4] = {w0.x, w0.y, w0.z, w0.w}, a1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int wd = 0; wd < 4; ++wd) {
            float2 k0[2], k1[2];
            i8x4_to_f2(a0[wd], k0[0], k0[1]);
            i8x4_to_f2(a1[wd], k1[0], k1[1]);
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
              const int cp = c * 8 + wd * 2 + hp;  // channel pair
#pragma unroll
              for (int g = 0; g < GRP; ++g) {
                const float2 qq = q2[cp * GRP + g];
                acc[0][g] = __ffma2_rn(k0[hp], qq, acc[0][g]);
                acc[1][g] = __ffma2_rn(k1[hp], qq, acc[1][g]);
              }
            }
          }
        }
      } else {
        // 32 codes (one swizzled chunk of packed INT4) per key per step
#pragma unroll 1
        for (int c = 0; c < C::kRow4 / 16; ++c) {
          const uint4 w0 = *reinterpret_cast<const uint4*>(kb + swz<C::kRow4>(lane, c));
          const uint4 w1 = *reinterpret_cast<const uint4*>(kb + swz<C::kRow4>(lane + 32, c));
          const uint32_t a0[4] = {w0.x, w0.y, w0.z, w0.w}, a1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int wd = 0; wd < 4; ++wd) {
            float2 k0[4], k1[4];
            i4x8_to_f2(a0[wd], k0);
            i4x8_to_f2(a1[wd], k1);
#pragma unroll
            for (int hp = 0; hp < 4; ++hp) {
              const int cp = c * 16 + wd * 4 + hp;
#pragma unroll
              for (int g = 0; g < GRP; ++g) {
                const float2 qq = q2[cp * GRP + g];
                acc[0][g] = __ffma2_rn(k0[hp], qq, acc[0][g]);
                acc[1][g] = __ffma2_rn(k1[hp], qq, acc[1][g]);
              }
            }
          }
        }
      }
      const float ks = (is8 ? __ldg(p.sk8 + tile) : __ldg(p.sk4 + tile)) * p.scale_log2;
      const float vs = is8 ? __ldg(p.sv8 + tile) : __ldg(p.sv4 + tile);
#pragma unroll
      for (int g = 0; g < GRP; ++g) {
        sc[0][g] = lane < nvalid ? (acc[0][g].x + acc[0][g].y) * ks : -INFINITY;
        sc[1][g] = lane + 32 < nvalid ? (acc[1][g].x + acc[1][g].y) * ks : -INFINITY;
      }
      if (is8) {
        softmax_pv(sc, vs, [&](int key, float2 (&v)[C::kCh / 2]) {
          if constexpr (D == 128) {  // channels 4*lane .. 4*lane+3
            const uint32_t w = *reinterpret_cast<const uint32_t*>(
                vb + swz<C::kRow8>(key, lane >> 2) + (lane & 3) * 4);
            i8x4_to_f2(w, v[0], v[1]);
          } else {  // D = 64: channels 2*lane, 2*lane+1
            const uint32_t w = *reinterpret_cast<const uint16_t*>(
                vb + swz<C::kRow8>(key, lane >> 3) + (lane & 7) * 2);
            float2 a, bb;
            i8x4_to_f2(w, a, bb);
            v[0] = a;
          }
        });
      } else {
        softmax_pv(sc, vs, [&](int key, float2 (&v)[C::kCh / 2]) {
          if constexpr (D == 128) {  // channels 4*lane .. 4*lane+3 = two packed bytes
            const uint32_t w = *reinterpret_cast<const uint16_t*>(
                vb + swz<C::kRow4>(key, lane >> 3) + (lane & 7) * 2);
            float2 f[4];
            i4x8_to_f2(w, f);
            v[0] = f[0];
            v[1] = f[1];
          } else {  // D = 64: channels 2*lane, 2*lane+1 = one packed byte
            const uint32_t w = *reinterpret_cast<const uint8_t*>(
                vb + swz<C::kRow4>(key, lane >> 4) + (lane & 15));
            float2 f[4];
            i4x8_to_f2(w, f);
            v[0] = f[0];
          }
        });
      }
      // stage s may be refilled once every lane of this warp is done with it
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + s * 8);
    }

    // ---- bf16 tail on the last split: tokens [0, tl) from the tail buffer, tl = new token
    if (ok && last && warp == 0) {
      const long long tbase = ((long long)b * p.Hkv + kvh) * p.tail_cap;
      const long long nbase = ((long long)b * p.Hkv + kvh) * D;
      for (int t0 = 0; t0 <= tl; t0 += kTile) {
        float sc[2][GRP];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int pos = t0 + lane + 32 * k;
          float2 acc[GRP];
#pragma unroll
          for (int g = 0; g < GRP; ++g) acc[g] = make_float2(0.0f, 0.0f);
          if (pos <= tl) {
            const uint16_t* kr = pos == tl ? p.k_new + nbase : p.k_tail + (tbase + pos) * D;
            for (int c = 0; c < D / 8; ++c) {
              const uint4 w = *reinterpret_cast<const uint4*>(kr + c * 8);
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int x = 0; x < 4; ++x) {
                const float2 kk = make_float2(__uint_as_float(ww[x] << 16),
                                              __uint_as_float(ww[x] & 0xFFFF0000u));
#pragma unroll
                for (int g = 0; g < GRP; ++g)
                  acc[g] = __ffma2_rn(kk, q2[(c * 4 + x) * GRP + g], acc[g]);
              }
            }
          }
#pragma unroll
          for (int g = 0; g < GRP; ++g)
            sc[k][g] = pos <= tl ? (acc[g].x + acc[g].y) * p.scale_log2 : -INFINITY;
        }
        softmax_pv(sc, 1.0f, [&](int key, float2 (&v)[C::kCh / 2]) {
          const int pos = t0 + key;
          if (pos > tl) {
#pragma unroll
            for (int k = 0; k < C::kCh / 2; ++k) v[k] = make_float2(0.0f, 0.0f);
            return;
          }
          const uint16_t* vr = pos == tl ? p.v_new + nbase : p.v_tail + (tbase + pos) * D;
#pragma unroll
          for (int k = 0; k < C::kCh / 2; ++k) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(vr + lane * C::kCh + 2 * k);
            v[k] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
          }
        });
      }
    }

    // ---- this warp's state into shared memory for the CTA merge
    float* rw = red + warp * GRP * (D + 2);
#pragma unroll
    for (int g = 0; g < GRP; ++g) {
#pragma unroll
      for (int k = 0; k < C::kCh / 2; ++k)
        *reinterpret_cast<float2*>(rw + g * (D + 2) + lane * C::kCh + 2 * k) = o2[g][k];
      if (lane == 0) {
        rw[g * (D + 2) + D] = m_run[g];
        rw[g * (D + 2) + D + 1] = l_run[g];
      }
    }
  }
  __syncthreads();
  // merge the consumer warps into this split's partial (m, l, o)
  for (int x = t; x < GRP * D; x += kDecThreads) {
    const int g = x / D, c = x % D;
    if (g >= grp) continue;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, red[(w * GRP + g) * (D + 2) + D]);
    float L = 0.0f, o = 0.0f;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) {
      const float* r = red + (w * GRP + g) * (D + 2);
      const float wt = r[D] == -INFINITY ? 0.0f : ex2(r[D] - M);
      L += r[D + 1] * wt;
      o += r[c] * wt;
    }
    const long long pi = ((long long)b * p.Hq + kvh * grp + g) * p.splits + split;
    p.part_o[pi * D + c] = o;
    if (c == 0) {
      p.part_ml[pi * 2] = M;
      p.part_ml[pi * 2 + 1] = L;
    }
  }
  if (t == 0 && *err) atomicOr(p.status, *err);
}

// One block per (sequence, query head): merge the splits' partials.
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  if (p.skip[b]) return;  // full tail: output and tail untouched
  const long long pi = (long long)bh * p.splits;
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, p.part_ml[(pi + s) * 2]);
  float L = 0.0f;
  for (int s = 0; s < p.splits; ++s) {
    const float m = p.part_ml[(pi + s) * 2];
    if (m != -INFINITY) L += p.part_ml[(pi + s) * 2 + 1] * ex2(m - M);
  }
  const float inv = L > 0.0f ? 1.0f / L : 0.0f;
  for (int c = threadIdx.x; c < p.d; c += blockDim.x) {
    float o = 0.0f;
    for (int s = 0; s < p.splits; ++s) {
      const float m = p.part_ml[(pi + s) * 2];
      if (m != -INFINITY) o += p.part_o[(pi + s) * p.d + c] * ex2(m - M);
    }
    const __nv_bfloat16 r = __float2bfloat16_rn(o * inv);
    p.out[(long long)bh * p.d + c] = *reinterpret_cast<const uint16_t*>(&r);
  }
  // only this block touches tail_len[b]; every split has read it already
  if (threadIdx.x == 0 && bh % p.Hq == 0) p.tail_len[b] += 1;
}

template <int D, int GRP>
cudaError_t launch_dec(const DecodeParams& p, const DecodeMaps& m, cudaStream_t s) {
  using C = DecCfg<D, GRP>;
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, GRP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.splits, p.Hkv, p.B);
  decode_split_kernel<D, GRP><<<grid, kDecThreads, C::kSmem, s>>>(p, m);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<p.B * p.Hq, 128, 0, s>>>(p);
  return cudaGetLastError();
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

int decode_splits(int B, int Hkv) {
  const int target = 2048;  // about seven waves of two CTAs per SM: a small tail
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
