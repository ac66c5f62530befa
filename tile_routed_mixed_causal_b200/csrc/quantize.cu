// quantize.cu -- per-(head, 64-token tile) symmetric INT8/INT4 (and FP8 E4M3) quantisation of
// Q, K and V (TriAttention abstract: the prefill prepares quantised keys and
// values; TileMix abstract: INT8 score tiles and INT8 K/V caches).
//
// One CTA per (tensor, head, tile): the 64 x d bf16 tile is read once with
// 16-byte loads into registers, the absolute maximum is reduced with warp
// shuffles, and the INT8 codes, packed INT4 codes, INT4 codes expanded to the
// int8 operand form (16 x code), FP8 E4M3 codes and their scales are written
// tile-major.  HBM-bound: 2*64*d bytes in, per requested format 64*d (INT8,
// expanded INT4, FP8) or 64*d/2 (packed INT4) bytes + 4 (scale) out.
// Arithmetic: s = fl32(amax / qmax) and code = rne(fl32(x / s)) with IEEE
// division (__fdiv_rn) and round-half-even conversion (__float2int_rn); FP8:
// sf = fl32(amax / 448) and the hardware's round-to-nearest-even, saturating
// conversion of fl32(x / sf) to E4M3.
#include "tra_device.cuh"
#include "tra_launch.h"

namespace tra {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }

// Two fp32 values to FP8 E4M3 codes (round to nearest even, saturating at +-448):
// byte 0 = lo, byte 1 = hi.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int D>
__global__ void __launch_bounds__(256) quantize_kernel(const QuantParams p) {
  constexpr int kChunks = D / 8;                 // 16-byte chunks per row
  constexpr int kPasses = kTile * kChunks / 256;  // chunks per thread
  __shared__ float red[8];

  const long long cta = blockIdx.x;
  int which = 0;
  while (which < 2 && cta >= p.cta_begin[which + 1]) ++which;
  const QuantTensor& t = p.t[which];
  const long long local = cta - p.cta_begin[which];
  const int h = (int)(local / p.ntiles);
  const int gt = (int)(local % p.ntiles);

  // sequence of this tile
  int b = 0, toff = 0;
  for (;; ++b) {
    const int nt = (p.cu[b + 1] - p.cu[b] + kTile - 1) / kTile;
    if (gt < toff + nt) break;
    toff += nt;
  }
  const int T = p.cu[b + 1] - p.cu[b];
  const int tt = gt - toff;
  const int H = t.H;

  uint4 v[kPasses];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const int f = i * 256 + threadIdx.x;
    const int r = f / kChunks, c = f % kChunks;
    const int tok = tt * kTile + r;
    if (tok < T) {
      const uint4* src = reinterpret_cast<const uint4*>(
          t.x + ((long long)(p.cu[b] + tok) * H + h) * D + c * 8);
      v[i] = __ldg(src);
    } else {
      v[i] = make_uint4(0, 0, 0, 0);
    }
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      amax = fmaxf(amax, fabsf(bf16_lo(w[j])));
      amax = fmaxf(amax, fabsf(bf16_hi(w[j])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);

  const float s8 = __fdiv_rn(amax, 127.0f);
  const float s4 = __fdiv_rn(amax, 7.0f);
  const float sf = __fdiv_rn(amax, 448.0f);  // FP8 E4M3: largest finite magnitude 448
  const long long tile_base = (long long)h * p.ntiles + gt;
  if (threadIdx.x == 0) {
    if (t.s8) t.s8[tile_base] = s8;
    if (t.s4) t.s4[tile_base] = s4;
    if (t.sf) t.sf[tile_base] = sf;
  }
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const int f = i * 256 + threadIdx.x;
    const int r = f / kChunks, c = f % kChunks;
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    float x[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[2 * j] = bf16_lo(w[j]);
      x[2 * j + 1] = bf16_hi(w[j]);
    }
    // rows past the sequence end were loaded as 0 and quantise to code 0
    if (t.x8) {
      const uint32_t flip = t.bias8 ? 0x80808080u : 0u;  // offset-binary: code + 128
      uint32_t o[2] = {0, 0};
#pragma unroll
      for (int j = 0; j < 8; ++j)
        o[j >> 2] |= (uint32_t)(quant_code(x[j], s8, 127) & 0xFF) << ((j & 3) * 8);
      o[0] ^= flip;
      o[1] ^= flip;
      *reinterpret_cast<uint2*>(t.x8 + (tile_base * kTile + r) * D + c * 8) = make_uint2(o[0], o[1]);
    }
    if (t.x4x) {  // INT4 codes as int8 operand values 16 x code (exact, |16 x code| <= 112)
      uint32_t o[2] = {0, 0};
#pragma unroll
      for (int j = 0; j < 8; ++j)
        o[j >> 2] |= (uint32_t)((quant_code(x[j], s4, 7) * 16) & 0xFF) << ((j & 3) * 8);
      *reinterpret_cast<uint2*>(t.x4x + (tile_base * kTile + r) * D + c * 8) = make_uint2(o[0], o[1]);
    }
    if (t.xf) {  // E4M3 of fl32(x / sf); a zero scale (all-zero tile) gives codes 0
      uint32_t o[2] = {0, 0};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t w2 = sf == 0.0f ? 0u : e4m3x2(__fdiv_rn(x[2 * j], sf), __fdiv_rn(x[2 * j + 1], sf));
        o[j >> 1] |= w2 << ((j & 1) * 16);
      }
      *reinterpret_cast<uint2*>(t.xf + (tile_base * kTile + r) * D + c * 8) = make_uint2(o[0], o[1]);
    }
    if (t.x4) {
      uint32_t o = 0;  // byte jj: channels 8c + 2jj (low nibble) and 8c + 2jj + 1
#pragma unroll
      for (int j = 0; j < 8; ++j) o |= (uint32_t)(quant_code(x[j], s4, 7) & 0x0F) << (j * 4);
      uint8_t* row = t.x4 + (tile_base * kTile + r) * (D / 2);
      if (!t.perm4) {
        *reinterpret_cast<uint32_t*>(row + c * 4) = o;
      } else {
        // decode order: in each 16-byte group m, byte 2g + e holds the byte that
        // row-major order keeps at 16m + 8e + g.  Chunks c and c ^ 2 (lanes t, t ^ 2)
        // fill the same 8 bytes, even positions from e = 0 and odd from e = 1.
        const uint32_t other = __shfl_xor_sync(0xffffffffu, o, 2);
        const int e = (c >> 1) & 1;
        const uint32_t w = e ? __byte_perm(o, other, 0x3726) : __byte_perm(o, other, 0x5140);
        *reinterpret_cast<uint32_t*>(row + 16 * (c >> 2) + 8 * (c & 1) + 4 * e) = w;
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize(const QuantParams& p, cudaStream_t s) {
  const long long ctas = p.cta_begin[3];
  if (ctas == 0) return cudaSuccess;
  if (ctas > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  if (p.d == 128)
    quantize_kernel<128><<<(unsigned)ctas, 256, 0, s>>>(p);
  else
    quantize_kernel<64><<<(unsigned)ctas, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace tra
