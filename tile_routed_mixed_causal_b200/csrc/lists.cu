// lists.cu -- precision-grouped traversal lists (TriAttention abstract: the
// per-head boundaries are expanded into traversals grouped by precision;
// TileMix abstract: routing bits packed into bitmasks, one bit per group of
// adjacent key tiles).
//
// One warp per CSR row.  Row lengths have closed forms in every mode (boundary
// rows keep min(qt+1, b2) tiles, bitmask rows keep all qt+1 causal tiles,
// decode-cache rows keep min(nt, max b2 of the group) or nt), so each warp
// computes its own row offset directly and the whole build is one launch with
// coalesced, warp-contiguous entry writes.
#include "tra_device.cuh"
#include "tra_launch.h"

namespace tra {
namespace {

// sum_{q=0}^{n-1} min(q+1, c)
__device__ __forceinline__ long long tri_capped(long long n, long long c) {
  if (n <= c) return n * (n + 1) / 2;
  return c * (c + 1) / 2 + (n - c) * c;
}

__device__ __forceinline__ int seq_tiles(const int32_t* cu, int b) {
  return (cu[b + 1] - cu[b] + kTile - 1) / kTile;
}

__device__ __forceinline__ long long warp_sum(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int group_max_b(const int32_t* b, int kvh, int grp) {
  int m = 0;
  for (int j = 0; j < grp; ++j) m = max(m, b[kvh * grp + j]);
  return m;
}

__global__ void __launch_bounds__(256) lists_kernel(const ListParams p) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row > p.rows) return;
  const long long cap_none = 1ll << 40;

  if (p.kind == TRA_LISTS_PREFILL) {
    if (row == p.rows) {  // final row_ptr entry = nnz
      long long tot = 0;
      for (long long i = lane; i < (long long)p.Hq * p.B; i += 32) {
        const int h = (int)(i / p.B), b = (int)(i % p.B);
        const long long c = p.mode != TRA_POLICY_BITMASK ? p.b2[h] : cap_none;
        tot += tri_capped(seq_tiles(p.cu, b), c);
      }
      tot = warp_sum(tot);
      if (lane == 0) p.row_ptr[row] = (int32_t)tot;
      return;
    }
    const int h = (int)(row / p.ntiles);
    const int gt = (int)(row % p.ntiles);
    int b = 0, toff = 0;
    for (;; ++b) {
      const int nt = seq_tiles(p.cu, b);
      if (gt < toff + nt) break;
      toff += nt;
    }
    const int qt = gt - toff;
    const long long c = p.mode != TRA_POLICY_BITMASK ? p.b2[h] : cap_none;
    // offset = all earlier heads + earlier sequences of this head + earlier rows
    long long off = 0;
    for (long long i = lane; i < (long long)h * p.B + b; i += 32) {
      const int hh = (int)(i / p.B), bb = (int)(i % p.B);
      const long long cc = p.mode != TRA_POLICY_BITMASK ? p.b2[hh] : cap_none;
      off += tri_capped(seq_tiles(p.cu, bb), cc);
    }
    off = warp_sum(off) + tri_capped(qt, c);
    if (lane == 0) p.row_ptr[row] = (int32_t)off;
    uint32_t* e = p.entries + off;
    if (p.mode == TRA_POLICY_BOUNDARY) {
      // the kept tiles qt-n+1 .. qt in distance bands: INT4 (farthest), then FP8, then
      // INT8 (nearest); written as the INT4 group, the INT8 group, the FP8 group
      const int n = min(qt + 1, p.b2[h]);
      const int n8 = min(qt + 1, p.b1[h]);
      const int nf = min(qt + 1, p.b8[h]) - n8;
      const int n4 = n - n8 - nf;
      for (int i = lane; i < n; i += 32) {
        const uint32_t kt = (uint32_t)(qt - n + 1 + i);
        if (i < n4)
          e[i] = ((uint32_t)TRA_PREC_INT4 << 28) | kt;
        else if (i < n4 + nf)
          e[n4 + n8 + (i - n4)] = ((uint32_t)TRA_PREC_FP8 << 28) | kt;
        else
          e[n4 + (i - n4 - nf)] = ((uint32_t)TRA_PREC_INT8 << 28) | kt;
      }
    } else if (p.mode == TRA_POLICY_MIXED) {
      // kept tiles qt-n+1 .. qt as under boundaries; a set bit promotes one to BF16.
      // Pass 1 counts the INT4 and INT8 tiles, pass 2 writes each group ascending.
      const int n = min(qt + 1, p.b2[h]);
      const int k0 = qt - n + 1;
      const uint32_t* words = p.bitmask + ((long long)h * p.ntiles + gt) * p.W;
      auto class_of = [&](int kt) -> int {  // 1 INT4, 2 INT8, 3 BF16
        const int g = kt / p.G;
        if ((__ldg(words + (g >> 5)) >> (g & 31)) & 1u) return TRA_PREC_BF16;
        return qt - kt < p.b1[h] ? TRA_PREC_INT8 : TRA_PREC_INT4;
      };
      int n4 = 0, n8 = 0;
      for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        const int cl = i < n ? class_of(k0 + i) : 0;
        n4 += __popc(__ballot_sync(0xffffffffu, cl == TRA_PREC_INT4));
        n8 += __popc(__ballot_sync(0xffffffffu, cl == TRA_PREC_INT8));
      }
      int c4 = 0, c8 = 0, c16 = 0;
      for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        const int cl = i < n ? class_of(k0 + i) : 0;
        const uint32_t m4 = __ballot_sync(0xffffffffu, cl == TRA_PREC_INT4);
        const uint32_t m8 = __ballot_sync(0xffffffffu, cl == TRA_PREC_INT8);
        const uint32_t m16 = __ballot_sync(0xffffffffu, cl == TRA_PREC_BF16);
        const uint32_t below = (1u << lane) - 1u;
        const uint32_t v = ((uint32_t)cl << 28) | (uint32_t)(k0 + i);
        if (cl == TRA_PREC_INT4) e[c4 + __popc(m4 & below)] = v;
        if (cl == TRA_PREC_INT8) e[n4 + c8 + __popc(m8 & below)] = v;
        if (cl == TRA_PREC_BF16) e[n4 + n8 + c16 + __popc(m16 & below)] = v;
        c4 += __popc(m4);
        c8 += __popc(m8);
        c16 += __popc(m16);
      }
    } else {
      const uint32_t* words = p.bitmask + ((long long)h * p.ntiles + gt) * p.W;
      // pass 1: number of INT8 (bit 0) tiles
      int n8 = 0;
      for (int base = 0; base <= qt; base += 32) {
        const int kt = base + lane;
        bool is8 = false;
        if (kt <= qt) {
          const int g = kt / p.G;
          is8 = ((__ldg(words + (g >> 5)) >> (g & 31)) & 1u) == 0;
        }
        n8 += __popc(__ballot_sync(0xffffffffu, is8));
      }
      // pass 2: INT8 tiles ascending at [0, n8), BF16 ascending after
      int c8 = 0, c16 = 0;
      for (int base = 0; base <= qt; base += 32) {
        const int kt = base + lane;
        bool valid = kt <= qt, is8 = false;
        if (valid) {
          const int g = kt / p.G;
          is8 = ((__ldg(words + (g >> 5)) >> (g & 31)) & 1u) == 0;
        }
        const uint32_t m8 = __ballot_sync(0xffffffffu, valid && is8);
        const uint32_t m16 = __ballot_sync(0xffffffffu, valid && !is8);
        const uint32_t below = (1u << lane) - 1u;
        if (valid) {
          if (is8)
            e[c8 + __popc(m8 & below)] = ((uint32_t)TRA_PREC_INT8 << 28) | (uint32_t)kt;
          else
            e[n8 + c16 + __popc(m16 & below)] = ((uint32_t)TRA_PREC_BF16 << 28) | (uint32_t)kt;
        }
        c8 += __popc(m8);
        c16 += __popc(m16);
      }
    }
    return;
  }

  // ---- decode-cache rows (b, kvh)
  const int grp = p.Hq / p.Hkv;
  auto row_count = [&](int bb, int kk) -> long long {
    const int nt = seq_tiles(p.cu, bb);
    if (p.mode == TRA_POLICY_BITMASK) return nt;
    return min(nt, group_max_b(p.b2, kk, grp));
  };
  long long off = 0;
  for (long long i = lane; i < row; i += 32) off += row_count((int)(i / p.Hkv), (int)(i % p.Hkv));
  off = warp_sum(off);
  if (lane == 0) p.row_ptr[row] = (int32_t)off;
  if (row == p.rows) return;
  const int b = (int)(row / p.Hkv), kvh = (int)(row % p.Hkv);
  const int nt = seq_tiles(p.cu, b);
  uint32_t* e = p.entries + off;
  if (p.mode != TRA_POLICY_BITMASK) {  // boundaries (mixed policies too); an FP8-band tile is cached as INT8
    const int n = min(nt, group_max_b(p.b2, kvh, grp));
    const int n8 = min(nt, group_max_b(p.b8, kvh, grp));
    for (int i = lane; i < n; i += 32) {
      const uint32_t prec = i < n - n8 ? TRA_PREC_INT4 : TRA_PREC_INT8;
      e[i] = (prec << 28) | (uint32_t)(nt - n + i);
    }
  } else {
    for (int i = lane; i < nt; i += 32) e[i] = ((uint32_t)TRA_PREC_INT8 << 28) | (uint32_t)i;
  }
}

}  // namespace

cudaError_t launch_lists(const ListParams& p, cudaStream_t s) {
  const long long warps = p.rows + 1;
  const long long blocks = (warps + 7) / 8;
  if (blocks > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  lists_kernel<<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace tra
