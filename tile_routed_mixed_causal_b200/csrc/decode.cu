// decode.cu -- one decode step over the compressed KV cache (TriAttention
// abstract: the K/V quantised during prefill become a compressed KV cache for
// decoding, which cuts the re-reading of the prompt; HyQuant, "How HyQuant
// works": dequantisation is done inside the attention kernel so it costs no
// extra memory pass).
//
// Split-K over the cached tiles of each (sequence, KV head): CTA (split, kvh, b)
// streams its share of the kept INT8/INT4 K/V tiles through a 4-deep ring of
// 1-D bulk copies (tiles are contiguous in the tile-major cache), dequantises
// in registers (K: one scale per tile applied to the integer dot product; V:
// the scale folded into P), and keeps one online-softmax state per query head
// of the GQA group, so every cached byte is read once per group.  The last
// split also covers the bf16 tail (earlier decode tokens plus the new one).
// A small combine kernel merges the splits' (m, l, o) and advances tail_len.
#include "tra_device.cuh"
#include "tra_launch.h"

namespace tra {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecStages = 4;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16f(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

template <int D, int GRP>
struct DecCfg {
  static constexpr int kParts = 4;                    // threads per key row in the score phase
  static constexpr int kPartCh = D / kParts;          // channels per part
  static constexpr int kQStride = kPartCh + 4;        // padded (bank-conflict free)
  static constexpr int kCg = D / 4;                   // 4-channel groups in the P*V phase
  static constexpr int kKs = kDecThreads / kCg;       // key subsets in the P*V phase
  static constexpr int kKeysPerSubset = kTile / kKs;
  static constexpr int kStageBytes = 2 * kTile * D;   // K + V codes (INT8 size)
  static constexpr int kRingBytes = kDecStages * kStageBytes;
  static constexpr int kRedBytes = kKs * GRP * D * 4;  // aliases the ring once it is drained
  static constexpr int kDynSmem = kRingBytes > kRedBytes ? kRingBytes : kRedBytes;
};

template <int D, int GRP>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const DecodeParams p) {
  using C = DecCfg<D, GRP>;
  extern __shared__ __align__(128) uint8_t dyn_smem[];
  uint8_t(*ring)[C::kStageBytes] = reinterpret_cast<uint8_t(*)[C::kStageBytes]>(dyn_smem);
  float(*red)[GRP][D] = reinterpret_cast<float(*)[GRP][D]>(dyn_smem);
  __shared__ __align__(16) float q_sm[GRP][C::kParts][C::kQStride];
  __shared__ float s_sm[GRP][kTile];
  __shared__ float p_sm[GRP][kTile];
  __shared__ float alpha_sm[GRP];
  __shared__ float ml_sm[GRP][2];
  __shared__ __align__(8) uint64_t full_bar[kDecStages];
  __shared__ int err_sm;

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x;
  const int grp = p.Hq / p.Hkv;
  const int seq0 = __ldg(p.cu + b);
  const int T = __ldg(p.cu + b + 1) - seq0;
  const int toff = seq_tile_offset(p.cu, b);
  const int tl = __ldg(p.tail_len + b);
  const bool tail_full = tl >= p.tail_cap;
  if (tail_full) {
    if (split == 0 && kvh == 0 && t == 0) atomicOr(p.status, TRA_DEV_TAIL_FULL);
    return;
  }
  const long long row = (long long)b * p.Hkv + kvh;
  const int rs = __ldg(p.row_ptr + row), re = __ldg(p.row_ptr + row + 1);
  const int n = re - rs;
  const int my0 = rs + (int)((long long)n * split / p.splits);
  const int my1 = rs + (int)((long long)n * (split + 1) / p.splits);
  const int ntile = my1 - my0;
  const bool last = split == p.splits - 1;

  // append the new token to the tail (split 0 only; nobody reads slot tl from the tail)
  if (split == 0) {
    const long long src = ((long long)b * p.Hkv + kvh) * D;
    const long long dst = (((long long)b * p.Hkv + kvh) * p.tail_cap + tl) * D;
    for (int c = t; c < D; c += kDecThreads) {
      p.k_tail[dst + c] = p.k_new[src + c];
      p.v_tail[dst + c] = p.v_new[src + c];
    }
  }
  // query heads of the group, fp32 in shared memory
  for (int x = t; x < GRP * D; x += kDecThreads) {
    const int g = x / D, c = x % D;
    float v = 0.0f;
    if (g < grp) v = bf16f(p.q[((long long)b * p.Hq + kvh * grp + g) * D + c]);
    q_sm[g][c / C::kPartCh][c % C::kPartCh] = v;
  }
  if (t < GRP) {
    ml_sm[t][0] = -INFINITY;
    ml_sm[t][1] = 0.0f;
  }
  if (t == 0) {
    err_sm = 0;
    for (int s = 0; s < kDecStages; ++s) mbar_init(smem_u32(&full_bar[s]), 1);
    fence_barrier_init();
  }
  __syncthreads();

  auto tile_info = [&](int idx, uint32_t& prec, int& kt) {
    const uint32_t e = __ldg(p.entries + my0 + idx);
    prec = e >> 28;
    kt = (int)(e & 0x0FFFFFFFu);
  };
  auto issue = [&](int idx) {
    uint32_t prec;
    int kt;
    tile_info(idx, prec, kt);
    const int s = idx % kDecStages;
    const long long tile = (long long)kvh * p.ntiles + toff + kt;
    const uint32_t bytes = prec == TRA_PREC_INT8 ? kTile * D : kTile * D / 2;
    const uint32_t bar = smem_u32(&full_bar[s]);
    mbar_arrive_expect_tx(bar, 2 * bytes);
    if (prec == TRA_PREC_INT8) {
      bulk_load(smem_u32(ring[s]), p.k8 + tile * kTile * D, bytes, bar);
      bulk_load(smem_u32(ring[s]) + kTile * D, p.v8 + tile * kTile * D, bytes, bar);
    } else {
      bulk_load(smem_u32(ring[s]), p.k4 + tile * kTile * D / 2, bytes, bar);
      bulk_load(smem_u32(ring[s]) + kTile * D, p.v4 + tile * kTile * D / 2, bytes, bar);
    }
  };
  if (t == 0)
    for (int i = 0; i < kDecStages && i < ntile; ++i) issue(i);

  // P*V accumulators: 4 channels x GRP heads for this thread's channel group
  const int cg = t % C::kCg, ks = t / C::kCg;
  float acc[GRP][4];
#pragma unroll
  for (int g = 0; g < GRP; ++g)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[g][c] = 0.0f;

  const int jk = t >> 2, part = t & 3;  // score phase: key row, channel part

  // one block of up to 64 keys: scores -> online softmax -> P*V
  auto process = [&](auto load_k, auto load_v, float kscale, float vscale, int nvalid) {
    // ---- scores
    float kv[C::kPartCh];
    load_k(jk, part * C::kPartCh, kv);
    float dot[GRP];
#pragma unroll
    for (int g = 0; g < GRP; ++g) {
      float a = 0.0f;
      const float4* qq = reinterpret_cast<const float4*>(&q_sm[g][part][0]);
#pragma unroll
      for (int c = 0; c < C::kPartCh; c += 4) {
        const float4 q4 = qq[c / 4];
        a = fmaf(q4.x, kv[c], a);
        a = fmaf(q4.y, kv[c + 1], a);
        a = fmaf(q4.z, kv[c + 2], a);
        a = fmaf(q4.w, kv[c + 3], a);
      }
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      dot[g] = a;
    }
    if (part == 0) {
#pragma unroll
      for (int g = 0; g < GRP; ++g)
        s_sm[g][jk] = jk < nvalid ? dot[g] * kscale : -INFINITY;
    }
    __syncthreads();
    // ---- online softmax, warp g owns head g
    const int w = t >> 5, ln = t & 31;
    if (w < GRP) {
      const float s0 = s_sm[w][ln], s1 = s_sm[w][ln + 32];
      float mt = fmaxf(s0, s1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
      const float m_old = ml_sm[w][0];
      const float m_new = fmaxf(m_old, mt);
      const float base = m_new == -INFINITY ? 0.0f : m_new;
      const float p0 = s0 == -INFINITY ? 0.0f : ex2(s0 - base);
      const float p1 = s1 == -INFINITY ? 0.0f : ex2(s1 - base);
      float ps = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      p_sm[w][ln] = p0 * vscale;
      p_sm[w][ln + 32] = p1 * vscale;
      __syncwarp();
      if (ln == 0) {
        const float alpha = m_old == -INFINITY ? 0.0f : ex2(m_old - base);
        alpha_sm[w] = alpha;
        ml_sm[w][0] = m_new;
        ml_sm[w][1] = ml_sm[w][1] * alpha + ps;
      }
    }
    __syncthreads();
    // ---- P*V
#pragma unroll
    for (int g = 0; g < GRP; ++g) {
      const float a = alpha_sm[g];
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[g][c] *= a;
    }
#pragma unroll 4
    for (int kk = 0; kk < C::kKeysPerSubset; ++kk) {
      const int key = ks * C::kKeysPerSubset + kk;
      float vv[4];
      load_v(key, cg * 4, vv);
#pragma unroll
      for (int g = 0; g < GRP; ++g) {
        const float pp = p_sm[g][key];
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[g][c] = fmaf(pp, vv[c], acc[g][c]);
      }
    }
    __syncthreads();
  };

  bool ok = true;
  for (int i = 0; i < ntile; ++i) {
    const int s = i % kDecStages;
    // one thread waits (bounded); the block barrier publishes the landed tile
    // and makes the decision uniform, so a timeout cannot split the block
    const bool landed = t == 0 ? mbar_wait(smem_u32(&full_bar[s]), (i / kDecStages) & 1, &err_sm)
                               : true;
    if (!__syncthreads_and(landed)) {
      ok = false;
      break;
    }
    uint32_t prec;
    int kt;
    tile_info(i, prec, kt);
    const long long tile = (long long)kvh * p.ntiles + toff + kt;
    const int nvalid = min(kTile, T - kt * kTile);
    const uint8_t* kbuf = ring[s];
    const uint8_t* vbuf = ring[s] + kTile * D;
    if (prec == TRA_PREC_INT8) {
      const float ksc = __ldg(p.sk8 + tile) * p.scale_log2;
      const float vsc = __ldg(p.sv8 + tile);
      process(
          [&](int key, int c0, float* out) {
            const int8_t* src = reinterpret_cast<const int8_t*>(kbuf + key * D + c0);
#pragma unroll
            for (int c = 0; c < C::kPartCh; c += 16) {
              const uint4 w = *reinterpret_cast<const uint4*>(src + c);
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int x = 0; x < 16; ++x) out[c + x] = (float)(int8_t)(ww[x >> 2] >> ((x & 3) * 8));
            }
          },
          [&](int key, int c0, float* out) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(vbuf + key * D + c0);
#pragma unroll
            for (int x = 0; x < 4; ++x) out[x] = (float)(int8_t)(w >> (x * 8));
          },
          ksc, vsc, nvalid);
    } else {
      const float ksc = __ldg(p.sk4 + tile) * p.scale_log2;
      const float vsc = __ldg(p.sv4 + tile);
      process(
          [&](int key, int c0, float* out) {
            // kPartCh codes = kPartCh/2 packed bytes, read as 32-bit words
            const uint32_t* src =
                reinterpret_cast<const uint32_t*>(kbuf + key * (D / 2) + c0 / 2);
#pragma unroll
            for (int y = 0; y < C::kPartCh / 8; ++y) {
              const uint2 e = expand_int4x8(src[y]);
#pragma unroll
              for (int x = 0; x < 8; ++x)
                out[y * 8 + x] = (float)(int8_t)((x < 4 ? e.x : e.y) >> ((x & 3) * 8));
            }
          },
          [&](int key, int c0, float* out) {
            const uint16_t w = *reinterpret_cast<const uint16_t*>(vbuf + key * (D / 2) + c0 / 2);
            const uint2 e = expand_int4x8((uint32_t)w);
#pragma unroll
            for (int x = 0; x < 4; ++x) out[x] = (float)(int8_t)(e.x >> (x * 8));
          },
          ksc, vsc, nvalid);
    }
    // stage s is free again (process ends with a block barrier)
    if (t == 0 && i + kDecStages < ntile) issue(i + kDecStages);
  }

  // ---- bf16 tail: positions [0, tl) from the tail buffer, position tl = the new token
  if (ok && last) {
    const long long tbase = ((long long)b * p.Hkv + kvh) * p.tail_cap;
    const long long nbase = ((long long)b * p.Hkv + kvh) * D;
    for (int t0 = 0; t0 <= tl; t0 += kTile) {
      const int nv = min(kTile, tl + 1 - t0);
      auto krow = [&](int key) -> const uint16_t* {
        const int pos = t0 + key;
        return pos == tl ? p.k_new + nbase : p.k_tail + (tbase + pos) * D;
      };
      auto vrow = [&](int key) -> const uint16_t* {
        const int pos = t0 + key;
        return pos == tl ? p.v_new + nbase : p.v_tail + (tbase + pos) * D;
      };
      process(
          [&](int key, int c0, float* out) {
            if (key < nv) {
              const uint16_t* src = krow(key) + c0;
#pragma unroll
              for (int c = 0; c < C::kPartCh; c += 8) {
                const uint4 w = *reinterpret_cast<const uint4*>(src + c);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                  out[c + 2 * x] = __uint_as_float(ww[x] << 16);
                  out[c + 2 * x + 1] = __uint_as_float(ww[x] & 0xFFFF0000u);
                }
              }
            } else {
#pragma unroll
              for (int c = 0; c < C::kPartCh; ++c) out[c] = 0.0f;
            }
          },
          [&](int key, int c0, float* out) {
            if (key < nv) {
              const uint2 w = *reinterpret_cast<const uint2*>(vrow(key) + c0);
              out[0] = __uint_as_float(w.x << 16);
              out[1] = __uint_as_float(w.x & 0xFFFF0000u);
              out[2] = __uint_as_float(w.y << 16);
              out[3] = __uint_as_float(w.y & 0xFFFF0000u);
            } else {
              out[0] = out[1] = out[2] = out[3] = 0.0f;
            }
          },
          p.scale_log2, 1.0f, nv);
    }
  }

  // ---- reduce the key subsets and write this split's partial (m, l, o)
#pragma unroll
  for (int g = 0; g < GRP; ++g)
#pragma unroll
    for (int c = 0; c < 4; ++c) red[ks][g][cg * 4 + c] = acc[g][c];
  __syncthreads();
  for (int x = t; x < GRP * D; x += kDecThreads) {
    const int g = x / D, c = x % D;
    if (g >= grp) continue;
    float sum = 0.0f;
#pragma unroll
    for (int k = 0; k < C::kKs; ++k) sum += red[k][g][c];
    const long long pi = ((long long)b * p.Hq + kvh * grp + g) * p.splits + split;
    p.part_o[pi * D + c] = sum;
    if (c == 0) {
      p.part_ml[pi * 2] = ml_sm[g][0];
      p.part_ml[pi * 2 + 1] = ml_sm[g][1];
    }
  }
  if (t == 0 && err_sm) atomicOr(p.status, err_sm);
}

__global__ void __launch_bounds__(256) decode_combine_kernel(const DecodeParams p) {
  const int b = blockIdx.x;
  const int tl = __ldg(p.tail_len + b);
  if (tl >= p.tail_cap) return;
  for (int x = threadIdx.x; x < p.Hq * p.d; x += blockDim.x) {
    const int h = x / p.d, c = x % p.d;
    const long long pi = ((long long)b * p.Hq + h) * p.splits;
    float M = -INFINITY;
    for (int s = 0; s < p.splits; ++s) M = fmaxf(M, p.part_ml[(pi + s) * 2]);
    float L = 0.0f, o = 0.0f;
    for (int s = 0; s < p.splits; ++s) {
      const float m = p.part_ml[(pi + s) * 2];
      if (m == -INFINITY) continue;
      const float w = ex2(m - M);
      L += p.part_ml[(pi + s) * 2 + 1] * w;
      o += p.part_o[(pi + s) * p.d + c] * w;
    }
    const __nv_bfloat16 r = __float2bfloat16_rn(L > 0.0f ? o / L : 0.0f);
    p.out[((long long)b * p.Hq + h) * p.d + c] = *reinterpret_cast<const uint16_t*>(&r);
  }
  __syncthreads();
  if (threadIdx.x == 0) p.tail_len[b] = tl + 1;  // every head of b has been written
}

template <int D, int GRP>
cudaError_t launch_dec(const DecodeParams& p, cudaStream_t s) {
  using C = DecCfg<D, GRP>;
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, GRP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kDynSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.splits, p.Hkv, p.B);
  decode_split_kernel<D, GRP><<<grid, kDecThreads, C::kDynSmem, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<p.B, 256, 0, s>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_dec_d(const DecodeParams& p, cudaStream_t s) {
  const int grp = p.Hq / p.Hkv;
  if (grp <= 1) return launch_dec<D, 1>(p, s);
  if (grp <= 2) return launch_dec<D, 2>(p, s);
  if (grp <= 4) return launch_dec<D, 4>(p, s);
  return launch_dec<D, 8>(p, s);
}

}  // namespace

int decode_splits(int B, int Hkv) {
  const int target = 4 * 148;  // about four CTAs per SM
  const int rows = B * Hkv;
  int s = (target + rows - 1) / rows;
  if (s < 1) s = 1;
  if (s > TRA_MAX_DECODE_SPLITS) s = TRA_MAX_DECODE_SPLITS;
  return s;
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t s) {
  return p.d == 128 ? launch_dec_d<128>(p, s) : launch_dec_d<64>(p, s);
}

}  // namespace tra
