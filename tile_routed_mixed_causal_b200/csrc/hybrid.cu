// hybrid.cu -- token selection and the prefill's mixed operands for the
// token-level hybrid (HyQuant Uses Hybrid Precision to Compress LLM Attention,
// "The observation behind the method" and "How HyQuant works": a small set of
// important key positions -- vertical lines in the attention map -- and a recent
// window keep high precision, the rest of the context is read from quantised
// storage).
//
// Selection: one CTA per (sequence, KV head).  The n = ceil(frac * T) positions of
// largest importance (ties to the earlier position) are found by a radix select
// over unique 64-bit keys (orderable importance bits above the complemented
// position), then written in ascending order, as a 64-bit mask per 64-token tile,
// and as a compact bf16 copy of their K and V rows; the last `window` prefix
// tokens are copied too.  Together these are the high-precision side of the
// hybrid KV cache that the decode reads beside the INT4 tiles.
//
// Mixed operands: one CTA per (tile, KV head) writes K and V rows that are the
// bf16 row of a selected token and the INT4 code row of any other, the form in
// which the hybrid prefill's tensor-core tiles read keys and values outside the
// window.
#include "tra_device.cuh"
#include "tra_launch.h"

namespace tra {
namespace {

constexpr int kSelThreads = 512;

// Monotone map of a float's bits to unsigned order (-0 taken as +0).
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Key of position j: larger importance first, then the earlier position.
__device__ __forceinline__ uint64_t sel_key(const float* imp, int Hkv, int seq0, int kvh, int j) {
  const uint32_t o = ordered_bits(__ldg(imp + (long long)(seq0 + j) * Hkv + kvh));
  return ((uint64_t)o << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) hybrid_select_kernel(const HybridSelectParams p) {
  __shared__ uint32_t hist[256];
  __shared__ uint64_t s_pref;
  __shared__ uint32_t s_want;
  __shared__ uint32_t warp_cnt[kSelThreads / 32];
  __shared__ int s_base;
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int seq0 = __ldg(p.cu + b);
  const int T = __ldg(p.cu + b + 1) - seq0;
  const int toff = seq_tile_offset(p.cu, b);
  const int nt = (T + kTile - 1) / kTile;
  long long nl = (long long)ceil(p.frac * (double)T);
  if (nl > T) nl = T;
  if (nl > p.cap) nl = p.cap;  // the host sized cap for every sequence; never exceeded
  const int n = (int)nl;
  if (kvh == 0 && t == 0) p.sel_count[b] = n;

  // ---- radix select of the n-th largest key, 8 bits at a time from the top
  if (t == 0) {
    s_pref = 0;
    s_want = (uint32_t)n;
  }
  __syncthreads();
  if (n > 0 && n < T) {
    for (int dg = 7; dg >= 0; --dg) {
      for (int i = t; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      const uint64_t pref = s_pref;
      const int hi_shift = 8 * (dg + 1);
      for (int j = t; j < T; j += kSelThreads) {
        const uint64_t k = sel_key(p.imp, p.Hkv, seq0, kvh, j);
        if (hi_shift == 64 || (k >> hi_shift) == (pref >> hi_shift))
          atomicAdd(&hist[(k >> (8 * dg)) & 0xFF], 1u);
      }
      __syncthreads();
      if (t == 0) {
        uint32_t want = s_want, cum = 0;
        int bin = 255;
        for (; bin > 0; --bin) {
          if (cum + hist[bin] >= want) break;
          cum += hist[bin];
        }
        s_want = want - cum;
        s_pref = pref | ((uint64_t)bin << (8 * dg));
      }
      __syncthreads();
    }
  }
  // selected: key >= kth (all when n = T, none when n = 0)
  const uint64_t kth = n == 0 ? ~0ull : (n >= T ? 0ull : s_pref);
  const bool none = n == 0;

  // ---- ascending positions, tile masks
  int* const pos_out = p.sel_pos + ((long long)b * p.Hkv + kvh) * p.cap;
  if (t == 0) s_base = 0;
  __syncthreads();
  for (int c0 = 0; c0 < nt * kTile; c0 += kSelThreads) {
    const int j = c0 + t;
    const bool sel = !none && j < T && sel_key(p.imp, p.Hkv, seq0, kvh, j) >= kth;
    const uint32_t bal = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    // warp w covers positions c0 + 32 w ..: the half (w & 1) of tile (c0 + 32 w) / 64
    if (lane == 0 && c0 + 32 * warp < nt * kTile) {
      uint32_t* m32 = reinterpret_cast<uint32_t*>(p.sel_mask + (long long)kvh * p.ntiles + toff +
                                                  (c0 + 32 * warp) / kTile);
      m32[warp & 1] = bal;
    }
    __syncthreads();
    int before = s_base;
    for (int w = 0; w < warp; ++w) before += warp_cnt[w];
    if (sel) pos_out[before + __popc(bal & ((1u << lane) - 1u))] = j;
    __syncthreads();
    if (t == 0) {
      int tot = 0;
      for (int w = 0; w < kSelThreads / 32; ++w) tot += warp_cnt[w];
      s_base += tot;
    }
    __syncthreads();
  }

  // ---- bf16 copies: selected rows, then the last `window` prefix tokens
  constexpr int kVec = D / 8;  // 16-byte chunks per row
  const long long dst0 = ((long long)b * p.Hkv + kvh) * p.cap;
  for (int x = t; x < n * kVec; x += kSelThreads) {
    const int i = x / kVec, c = x % kVec;
    const long long src = ((long long)(seq0 + pos_out[i]) * p.Hkv + kvh) * D + c * 8;
    const long long dst = (dst0 + i) * D + c * 8;
    *reinterpret_cast<uint4*>(p.k_sel + dst) = __ldg(reinterpret_cast<const uint4*>(p.k + src));
    *reinterpret_cast<uint4*>(p.v_sel + dst) = __ldg(reinterpret_cast<const uint4*>(p.v + src));
  }
  const long long w0 = ((long long)b * p.Hkv + kvh) * p.window;
  for (int x = t; x < p.window * kVec; x += kSelThreads) {
    const int w = x / kVec, c = x % kVec;
    const int j = T - p.window + w;
    const long long dst = (w0 + w) * D + c * 8;
    uint4 kk = make_uint4(0, 0, 0, 0), vv = kk;
    if (j >= 0) {
      const long long src = ((long long)(seq0 + j) * p.Hkv + kvh) * D + c * 8;
      kk = __ldg(reinterpret_cast<const uint4*>(p.k + src));
      vv = __ldg(reinterpret_cast<const uint4*>(p.v + src));
    }
    *reinterpret_cast<uint4*>(p.k_win + dst) = kk;
    *reinterpret_cast<uint4*>(p.v_win + dst) = vv;
  }
}

// One CTA per (tile, KV head): the tile's 64 rows of K and V, 16 bytes per load,
// each row copied as is when its token is selected and otherwise replaced by its INT4
// codes (exact small integers in bf16).  HBM-bound: 2 * 64 * d * 2 bytes in and out
// per tile.
template <int D>
__global__ void __launch_bounds__(256) hybrid_mix_kernel(const HybridMixParams p) {
  constexpr int kChunks = D / 8;                 // 16-byte chunks per row
  constexpr int kPasses = kTile * kChunks / 256;  // chunks per thread
  const int gt = blockIdx.x, h = blockIdx.y;
  int b = 0, toff = 0;
  for (;; ++b) {
    const int nt = (__ldg(p.cu + b + 1) - __ldg(p.cu + b) + kTile - 1) / kTile;
    if (gt < toff + nt) break;
    toff += nt;
  }
  const int seq0 = __ldg(p.cu + b);
  const int T = __ldg(p.cu + b + 1) - seq0;
  const int tt = gt - toff;
  const long long tile = (long long)h * p.ntiles + gt;
  const float sk = __ldg(p.sk4 + tile), sv = __ldg(p.sv4 + tile);
  const uint64_t sel = __ldg(reinterpret_cast<const unsigned long long*>(p.sel_mask) + tile);
#pragma unroll
  for (int i = 0; i < kPasses; ++i) {
    const int f = i * 256 + threadIdx.x;
    const int r = f / kChunks, c = f % kChunks;
    const int tok = tt * kTile + r;
    if (tok >= T) continue;
    const long long off = ((long long)(seq0 + tok) * p.Hkv + h) * D + c * 8;
    uint4 kk = __ldg(reinterpret_cast<const uint4*>(p.k + off));
    uint4 vv = __ldg(reinterpret_cast<const uint4*>(p.v + off));
    if (!((sel >> r) & 1ull)) {
      auto codes = [](uint4 w, float s) {
        uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float lo = __uint_as_float(a[j] << 16), hi = __uint_as_float(a[j] & 0xFFFF0000u);
          const __nv_bfloat162 q2 = __floats2bfloat162_rn((float)quant_code(lo, s, 7),
                                                          (float)quant_code(hi, s, 7));
          a[j] = *reinterpret_cast<const uint32_t*>(&q2);
        }
        return make_uint4(a[0], a[1], a[2], a[3]);
      };
      kk = codes(kk, sk);
      vv = codes(vv, sv);
    }
    *reinterpret_cast<uint4*>(p.k_mix + off) = kk;
    *reinterpret_cast<uint4*>(p.v_mix + off) = vv;
  }
}

}  // namespace

cudaError_t launch_hybrid_mix(const HybridMixParams& p, cudaStream_t s) {
  if (p.ntiles == 0 || p.Hkv == 0) return cudaSuccess;
  dim3 grid(p.ntiles, p.Hkv);
  if (p.d == 128)
    hybrid_mix_kernel<128><<<grid, 256, 0, s>>>(p);
  else
    hybrid_mix_kernel<64><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_hybrid_select(const HybridSelectParams& p, cudaStream_t s) {
  dim3 grid(p.Hkv, p.B);
  if (p.d == 128)
    hybrid_select_kernel<128><<<grid, kSelThreads, 0, s>>>(p);
  else
    hybrid_select_kernel<64><<<grid, kSelThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace tra
