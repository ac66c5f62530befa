// tra_api.cu -- host side of the C ABI declared in include/tra.h: argument
// validation, closed-form sizes, TMA tensor-map construction and the launches.
// Every check happens before any launch; nothing here allocates device memory
// or synchronises the device.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#ifndef TRA_NO_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

#include "../../include/tra.h"
#include "tra_launch.h"

namespace {

// A named NVTX range around an ABI call (what a profiler timeline shows for it);
// free when no profiler is attached.  Build with -DTRA_NO_NVTX to leave it out.
struct CallRange {
#ifndef TRA_NO_NVTX
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
#else
  explicit CallRange(const char*) {}
#endif
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

thread_local std::string g_last_error;

tra_status fail(tra_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

tra_status ok() {
  g_last_error.clear();
  return TRA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ceil_tiles(int64_t T) { return (T + TRA_TILE - 1) / TRA_TILE; }

// Validates a shape; fills ntiles, ntok and the largest per-sequence tile count.
tra_status check_shape(const tra_shape* s, int64_t* ntiles, int64_t* ntok, int64_t* nt_max) {
  if (!s) return fail(TRA_ERR_INVALID, "shape is NULL");
  if (s->B < 1) return fail(TRA_ERR_INVALID, "B must be >= 1 (got %d)", s->B);
  if (s->Hq < 1 || s->Hkv < 1) return fail(TRA_ERR_INVALID, "Hq and Hkv must be >= 1");
  if (s->Hq % s->Hkv) return fail(TRA_ERR_INVALID, "Hq (%d) must be a multiple of Hkv (%d)", s->Hq, s->Hkv);
  if (s->Hq > TRA_MAX_HEADS) return fail(TRA_ERR_UNSUPPORTED, "Hq > %d", TRA_MAX_HEADS);
  if (s->d != 64 && s->d != 128) return fail(TRA_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", s->d);
  if (!s->cu_seqlens_host || !s->cu_seqlens_dev) return fail(TRA_ERR_INVALID, "cu_seqlens (host and device) required");
  if (reinterpret_cast<uintptr_t>(s->cu_seqlens_dev) & 3u) return fail(TRA_ERR_INVALID, "cu_seqlens_dev misaligned");
  if (s->cu_seqlens_host[0] != 0) return fail(TRA_ERR_INVALID, "cu_seqlens[0] must be 0");
  int64_t t = 0, m = 0;
  for (int b = 0; b < s->B; ++b) {
    const int64_t L = (int64_t)s->cu_seqlens_host[b + 1] - s->cu_seqlens_host[b];
    if (L < 0) return fail(TRA_ERR_INVALID, "cu_seqlens not non-decreasing at %d", b);
    t += ceil_tiles(L);
    if (ceil_tiles(L) > m) m = ceil_tiles(L);
  }
  if (t * TRA_TILE * (int64_t)s->Hq > (1ll << 31) * 64) return fail(TRA_ERR_UNSUPPORTED, "problem too large");
  if (ntiles) *ntiles = t;
  if (ntok) *ntok = s->cu_seqlens_host[s->B];
  if (nt_max) *nt_max = m;
  return TRA_OK;
}

// sum_{q < n} min(q + 1, c)
int64_t tri_capped(int64_t n, int64_t c) {
  if (n <= c) return n * (n + 1) / 2;
  return c * (c + 1) / 2 + (n - c) * c;
}

bool uses_boundaries(const tra_policy* p) { return p->mode != TRA_POLICY_BITMASK; }
bool uses_bitmask(const tra_policy* p) { return p->mode != TRA_POLICY_BOUNDARY; }

tra_status check_policy(const tra_shape* s, const tra_policy* p, int64_t nt_max) {
  if (!p) return fail(TRA_ERR_INVALID, "policy is NULL");
  if (p->mode != TRA_POLICY_BOUNDARY && p->mode != TRA_POLICY_BITMASK && p->mode != TRA_POLICY_MIXED)
    return fail(TRA_ERR_INVALID, "unknown policy mode %d", p->mode);
  if (uses_boundaries(p)) {
    if (!p->b1 || !p->b2) return fail(TRA_ERR_INVALID, "boundary policy needs host b1 and b2");
    for (int h = 0; h < s->Hq; ++h) {
      if (p->b1[h] < 1) return fail(TRA_ERR_INVALID, "b1[%d] = %d < 1", h, p->b1[h]);
      if (p->b2[h] < p->b1[h]) return fail(TRA_ERR_INVALID, "b2[%d] = %d < b1 = %d", h, p->b2[h], p->b1[h]);
    }
  }
  if (p->b8) {
    if (p->mode != TRA_POLICY_BOUNDARY)
      return fail(TRA_ERR_UNSUPPORTED, "the FP8 band (b8) is supported under boundary policies only");
    for (int h = 0; h < s->Hq; ++h)
      if (p->b8[h] < p->b1[h] || p->b8[h] > p->b2[h])
        return fail(TRA_ERR_INVALID, "need b1 <= b8 <= b2 (head %d: %d, %d, %d)", h, p->b1[h],
                    p->b8[h], p->b2[h]);
  }
  if (uses_bitmask(p)) {
    if (p->G < 1) return fail(TRA_ERR_INVALID, "G must be >= 1 (got %d)", p->G);
    if (p->W < 1) return fail(TRA_ERR_INVALID, "W must be >= 1");
    const int64_t groups = (nt_max + p->G - 1) / p->G;
    if ((int64_t)p->W * 32 < groups)
      return fail(TRA_ERR_INVALID, "W = %d words cannot hold %lld groups", p->W, (long long)groups);
  }
  return TRA_OK;
}

bool policy_has_int4(const tra_shape* s, const tra_policy* p) {
  if (!uses_boundaries(p)) return false;
  for (int h = 0; h < s->Hq; ++h)
    if (p->b2[h] > (p->b8 ? p->b8[h] : p->b1[h])) return true;
  return false;
}

bool policy_has_fp8(const tra_shape* s, const tra_policy* p) {
  if (p->mode != TRA_POLICY_BOUNDARY || !p->b8) return false;
  for (int h = 0; h < s->Hq; ++h)
    if (p->b8[h] > p->b1[h]) return true;
  return false;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// Tile-major codes viewed as 2-D: row_bytes per row (a row of a tile), `rows`
// rows; the swizzle span equals the row (128, 64 or 32 bytes).
bool map_i8(CUtensorMap* m, const void* base, int row_bytes, int64_t rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapSwizzle sw = row_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_32B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [ntok][H][d] viewed as 3-D (d, H, ntok); boxes of 64 channels x 1 head x box_rows tokens.
bool map_bf16(CUtensorMap* m, const void* base, int d, int H, int64_t ntok, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)ntok};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

tra_status cuda_fail(cudaError_t e, const char* what) {
  return fail(TRA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

namespace tra {
tra_status report_error(tra_status st, const char* msg) { return fail(st, "%s", msg); }
}  // namespace tra

extern "C" {

const char* tra_last_error(void) { return g_last_error.c_str(); }

const char* tra_version(void) { return "tile_routed_mixed_causal_b200 0.1 (sm_100a)"; }

int64_t tra_num_tiles(const tra_shape* shape) {
  int64_t nt = 0;
  if (check_shape(shape, &nt, nullptr, nullptr) != TRA_OK) return -1;
  return nt;
}

size_t tra_qtiles_bytes(const tra_shape* shape, uint32_t formats) {
  int64_t nt = 0;
  if (check_shape(shape, &nt, nullptr, nullptr) != TRA_OK) return 0;
  const size_t d = shape->d;
  size_t total = 0;
  // codes of each format; scales once per (tensor, precision): Q4X / K4X share the
  // INT4 scales of Q4 / K4
  const struct { uint32_t bit, scale_bits; int H; size_t per_row; } f[10] = {
      {TRA_FMT_Q8, TRA_FMT_Q8, shape->Hq, d},
      {TRA_FMT_Q4, TRA_FMT_Q4 | TRA_FMT_Q4X, shape->Hq, d / 2},
      {TRA_FMT_K8, TRA_FMT_K8, shape->Hkv, d},
      {TRA_FMT_K4, TRA_FMT_K4 | TRA_FMT_K4X, shape->Hkv, d / 2},
      {TRA_FMT_V8, TRA_FMT_V8, shape->Hkv, d},
      {TRA_FMT_V4, TRA_FMT_V4, shape->Hkv, d / 2},
      {TRA_FMT_Q4X, 0, shape->Hq, d},
      {TRA_FMT_K4X, 0, shape->Hkv, d},
      {TRA_FMT_Q8F, TRA_FMT_Q8F, shape->Hq, d},
      {TRA_FMT_K8F, TRA_FMT_K8F, shape->Hkv, d}};
  for (const auto& x : f) {
    if (formats & x.bit) total += round256((size_t)x.H * nt * TRA_TILE * x.per_row);
    if (formats & x.scale_bits) total += round256((size_t)x.H * nt * 4);
  }
  return total;
}

tra_status quantize_qkv_tiles(const tra_shape* shape, const uint16_t* q, const uint16_t* k,
                              const uint16_t* v, const tra_qtiles* out, void* stream) {
  const CallRange range("tra::quantize_qkv_tiles");
  int64_t nt = 0, ntok = 0;
  tra_status st = check_shape(shape, &nt, &ntok, nullptr);
  if (st != TRA_OK) return st;
  if (!out) return fail(TRA_ERR_INVALID, "out is NULL");
  const uint32_t f = out->formats;
  if (f & ~0x3FFu) return fail(TRA_ERR_INVALID, "unknown format bits 0x%x", f);
  tra::QuantParams p{};
  const uint16_t* src[3] = {q, k, v};
  const int H[3] = {shape->Hq, shape->Hkv, shape->Hkv};
  int8_t* o8[3] = {out->q8, out->k8, out->v8};
  uint8_t* o4[3] = {out->q4, out->k4, out->v4};
  int8_t* o4x[3] = {out->q4x, out->k4x, nullptr};
  const uint32_t fx[3] = {TRA_FMT_Q4X, TRA_FMT_K4X, 0u};
  uint8_t* of[3] = {out->q8f, out->k8f, nullptr};
  float* sfp[3] = {out->sqf, out->skf, nullptr};
  const uint32_t ff[3] = {TRA_FMT_Q8F, TRA_FMT_K8F, 0u};
  float* s8[3] = {out->sq8, out->sk8, out->sv8};
  float* s4[3] = {out->sq4, out->sk4, out->sv4};
  const char* nm[3] = {"q", "k", "v"};
  p.cta_begin[0] = 0;
  for (int i = 0; i < 3; ++i) {
    const bool want8 = f & (TRA_FMT_Q8 << (2 * i));
    const bool wantp = f & (TRA_FMT_Q4 << (2 * i));  // packed INT4
    const bool wantx = (f & fx[i]) != 0;              // INT4 as int8 16 x code
    const bool want4 = wantp || wantx;
    const bool wantf = (f & ff[i]) != 0;             // FP8 E4M3
    tra::QuantTensor& t = p.t[i];
    t = tra::QuantTensor{};
    if (want8 || want4 || wantf) {
      if (!src[i]) return fail(TRA_ERR_INVALID, "%s is NULL but its formats are requested", nm[i]);
      if (!aligned16(src[i])) return fail(TRA_ERR_INVALID, "%s not 16-byte aligned", nm[i]);
      if (want8 && (!o8[i] || !s8[i] || !aligned16(o8[i]) || !aligned16(s8[i])))
        return fail(TRA_ERR_INVALID, "%s8 codes/scales missing or misaligned", nm[i]);
      if (want4 && (!s4[i] || !aligned16(s4[i])))
        return fail(TRA_ERR_INVALID, "%s4 scales missing or misaligned", nm[i]);
      if (wantp && (!o4[i] || !aligned16(o4[i])))
        return fail(TRA_ERR_INVALID, "%s4 codes missing or misaligned", nm[i]);
      if (wantx && (!o4x[i] || !aligned16(o4x[i])))
        return fail(TRA_ERR_INVALID, "%s4x codes missing or misaligned", nm[i]);
      if (wantf && (!of[i] || !sfp[i] || !aligned16(of[i]) || !aligned16(sfp[i])))
        return fail(TRA_ERR_INVALID, "%s8f codes/scales missing or misaligned", nm[i]);
      t.x = src[i];
      t.H = H[i];
      t.x8 = want8 ? o8[i] : nullptr;
      t.s8 = want8 ? s8[i] : nullptr;
      t.x4 = wantp ? o4[i] : nullptr;
      t.x4x = wantx ? o4x[i] : nullptr;
      t.perm4 = i == 2;  // V4 is read only by the decode, in its MMA fragment order
      t.bias8 = i == 2;  // so is V8, kept offset-binary for its f16 conversion
      t.s4 = want4 ? s4[i] : nullptr;
      t.xf = wantf ? of[i] : nullptr;
      t.sf = wantf ? sfp[i] : nullptr;
    }
    p.cta_begin[i + 1] = p.cta_begin[i] + (t.x ? (long long)t.H * nt : 0);
  }
  p.cu = shape->cu_seqlens_dev;
  p.B = shape->B;
  p.d = shape->d;
  p.ntiles = (int)nt;
  if (nt == 0) return ok();
  cudaError_t e = tra::launch_quantize(p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return ok();
}

tra_status tra_tile_lists_size(const tra_shape* shape, const tra_policy* policy, int32_t list_kind,
                               int64_t* rows, int64_t* nnz) {
  int64_t nt = 0, nt_max = 0;
  tra_status st = check_shape(shape, &nt, nullptr, &nt_max);
  if (st != TRA_OK) return st;
  st = check_policy(shape, policy, nt_max);
  if (st != TRA_OK) return st;
  if (!rows || !nnz) return fail(TRA_ERR_INVALID, "rows/nnz outputs are NULL");
  const int32_t* cu = shape->cu_seqlens_host;
  int64_t total = 0;
  if (list_kind == TRA_LISTS_PREFILL) {
    *rows = (int64_t)shape->Hq * nt;
    for (int h = 0; h < shape->Hq; ++h)
      for (int b = 0; b < shape->B; ++b) {
        const int64_t n = ceil_tiles(cu[b + 1] - cu[b]);
        total += tri_capped(n, uses_boundaries(policy) ? policy->b2[h] : (1ll << 40));
      }
  } else if (list_kind == TRA_LISTS_DECODE_CACHE) {
    *rows = (int64_t)shape->B * shape->Hkv;
    const int grp = shape->Hq / shape->Hkv;
    for (int b = 0; b < shape->B; ++b) {
      const int64_t n = ceil_tiles(cu[b + 1] - cu[b]);
      for (int kvh = 0; kvh < shape->Hkv; ++kvh) {
        if (!uses_boundaries(policy)) {
          total += n;
          continue;
        }
        int64_t m = 0;
        for (int j = 0; j < grp; ++j) m = std::max<int64_t>(m, policy->b2[kvh * grp + j]);
        total += std::min(n, m);
      }
    }
  } else {
    return fail(TRA_ERR_INVALID, "unknown list kind %d", list_kind);
  }
  if (total >= (1ll << 31)) return fail(TRA_ERR_UNSUPPORTED, "list has %lld entries (> int32)", (long long)total);
  *nnz = total;
  return ok();
}

tra_status build_tile_lists(const tra_shape* shape, const tra_policy* policy, int32_t list_kind,
                            int32_t* row_ptr, int64_t row_ptr_len, uint32_t* entries,
                            int64_t entries_cap, void* stream) {
  const CallRange range("tra::build_tile_lists");
  int64_t rows = 0, nnz = 0;
  tra_status st = tra_tile_lists_size(shape, policy, list_kind, &rows, &nnz);
  if (st != TRA_OK) return st;
  if (!row_ptr || (!entries && nnz > 0)) return fail(TRA_ERR_INVALID, "row_ptr/entries NULL");
  if (!aligned16(row_ptr) || (entries && !aligned16(entries)))
    return fail(TRA_ERR_INVALID, "row_ptr/entries not 16-byte aligned");
  if (row_ptr_len < rows + 1) return fail(TRA_ERR_BUFFER, "row_ptr needs %lld entries", (long long)(rows + 1));
  if (entries_cap < nnz) return fail(TRA_ERR_BUFFER, "entries needs %lld entries", (long long)nnz);
  if (uses_bitmask(policy) && list_kind == TRA_LISTS_PREFILL) {
    if (!policy->bitmask_dev || (reinterpret_cast<uintptr_t>(policy->bitmask_dev) & 3u))
      return fail(TRA_ERR_INVALID, "bitmask_dev NULL or misaligned");
  }
  int64_t nt = tra_num_tiles(shape);
  tra::ListParams p;
  memset(&p, 0, sizeof p);
  p.cu = shape->cu_seqlens_dev;
  p.B = shape->B;
  p.Hq = shape->Hq;
  p.Hkv = shape->Hkv;
  p.ntiles = (int)nt;
  p.mode = policy->mode;
  p.kind = list_kind;
  p.bitmask = policy->bitmask_dev;
  p.G = policy->G;
  p.W = policy->W;
  p.row_ptr = row_ptr;
  p.entries = entries;
  p.rows = rows;
  if (uses_boundaries(policy))
    for (int h = 0; h < shape->Hq; ++h) {
      p.b1[h] = policy->b1[h];
      p.b2[h] = policy->b2[h];
      p.b8[h] = policy->b8 ? policy->b8[h] : policy->b1[h];
    }
  cudaError_t e = tra::launch_lists(p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lists launch");
  return ok();
}

tra_status routed_attention_prefill(const tra_shape* shape, const tra_policy* policy,
                                    const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                    const tra_qtiles* tiles, const int32_t* row_ptr,
                                    const uint32_t* entries, float softmax_scale, uint16_t* out,
                                    float* lse, const int32_t* dump_coords, int32_t n_dump,
                                    int32_t* dump_out, int32_t* status_dev, void* stream) {
  const CallRange range("tra::routed_attention_prefill");
  int64_t nt = 0, ntok = 0, nt_max = 0;
  tra_status st = check_shape(shape, &nt, &ntok, &nt_max);
  if (st != TRA_OK) return st;
  st = check_policy(shape, policy, nt_max);
  if (st != TRA_OK) return st;
  if (!q || !k || !v || !out || !tiles || !row_ptr || !entries || !status_dev)
    return fail(TRA_ERR_INVALID, "q, k, v, out, tiles, row_ptr, entries and status are required");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (lse && !aligned16(lse)))
    return fail(TRA_ERR_INVALID, "q/k/v/out/lse must be 16-byte aligned");
  const uint32_t need8 = TRA_FMT_Q8 | TRA_FMT_K8;
  if ((tiles->formats & need8) != need8 || !tiles->q8 || !tiles->k8 || !tiles->sq8 || !tiles->sk8)
    return fail(TRA_ERR_INVALID, "prefill needs Q8 and K8 tiles");
  if (!aligned16(tiles->q8) || !aligned16(tiles->k8)) return fail(TRA_ERR_INVALID, "Q8/K8 misaligned");
  const bool has4 = policy_has_int4(shape, policy);
  if (has4) {
    const uint32_t need4 = TRA_FMT_Q4X | TRA_FMT_K4X;
    if ((tiles->formats & need4) != need4 || !tiles->q4x || !tiles->k4x || !tiles->sq4 || !tiles->sk4)
      return fail(TRA_ERR_INVALID,
                  "the policy has INT4 tiles: Q4X and K4X tiles (INT4 as int8 operands) are required");
    if (!aligned16(tiles->q4x) || !aligned16(tiles->k4x)) return fail(TRA_ERR_INVALID, "Q4X/K4X misaligned");
  }
  const bool hasf = policy_has_fp8(shape, policy);
  if (hasf) {
    const uint32_t needf = TRA_FMT_Q8F | TRA_FMT_K8F;
    if ((tiles->formats & needf) != needf || !tiles->q8f || !tiles->k8f || !tiles->sqf || !tiles->skf)
      return fail(TRA_ERR_INVALID, "the policy has an FP8 band: Q8F and K8F tiles are required");
    if (!aligned16(tiles->q8f) || !aligned16(tiles->k8f)) return fail(TRA_ERR_INVALID, "Q8F/K8F misaligned");
  }
  if (nt_max >= (1ll << 24)) return fail(TRA_ERR_UNSUPPORTED, "a sequence has more than 2^24 tiles");
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale))
    return fail(TRA_ERR_INVALID, "softmax_scale must be positive and finite");
  if (n_dump < 0 || n_dump > TRA_MAX_DUMP) return fail(TRA_ERR_INVALID, "n_dump must be in [0, %d]", TRA_MAX_DUMP);
  if (n_dump > 0 && (!dump_coords || !dump_out)) return fail(TRA_ERR_INVALID, "dump buffers required");
  if (ntok == 0 || nt == 0) return ok();
  tra::PrefillParams p{};
  p.cu = shape->cu_seqlens_dev;
  p.B = shape->B;
  p.Hq = shape->Hq;
  p.Hkv = shape->Hkv;
  p.d = shape->d;
  p.ntiles = (int)nt;
  p.mode = hasf ? tra::kPrefillModeBoundaryF8 : policy->mode;
  p.has_int4 = policy_has_int4(shape, policy) ? 1 : 0;
  p.jmax = (int)((nt_max + 1) / 2);
  p.row_ptr = row_ptr;
  p.entries = entries;
  p.sq8 = tiles->sq8;
  p.sq4 = tiles->sq4;
  p.sk8 = tiles->sk8;
  p.sk4 = tiles->sk4;
  p.sqf = hasf ? tiles->sqf : nullptr;
  p.skf = hasf ? tiles->skf : nullptr;
  if (policy->mode == TRA_POLICY_BOUNDARY)
    for (int h = 0; h < shape->Hq; ++h) {
      p.b1[h] = policy->b1[h];
      p.b8[h] = policy->b8 ? policy->b8[h] : policy->b1[h];
    }
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out;
  p.lse = lse;
  p.dump_coords = dump_coords;
  p.n_dump = n_dump;
  p.dump_out = dump_out;
  p.status = status_dev;
  tra::PrefillMaps m;
  memset(&m, 0, sizeof m);
  const int d = shape->d;
  const int64_t qrows = (int64_t)shape->Hq * nt * TRA_TILE, krows = (int64_t)shape->Hkv * nt * TRA_TILE;
  bool good = map_i8(&m.q8, tiles->q8, d, qrows, 128) && map_i8(&m.k8, tiles->k8, d, krows, 64) &&
              (!has4 || (map_i8(&m.q4x, tiles->q4x, d, qrows, 128) &&
                         map_i8(&m.k4x, tiles->k4x, d, krows, 64))) &&
              map_bf16(&m.qb, q, d, shape->Hq, ntok, 128) &&
              map_bf16(&m.kb, k, d, shape->Hkv, ntok, 64) &&
              map_bf16(&m.vb, v, d, shape->Hkv, ntok, 64) &&
              (!hasf || (map_i8(&m.qf8, tiles->q8f, d, qrows, 128) &&
                         map_i8(&m.kf8, tiles->k8f, d, krows, 64)));
  if (!good) return fail(TRA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  cudaError_t e = tra::launch_prefill(p, m, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return ok();
}

// Decode workspace: arrival counters first, in a region of fixed size for every
// shape up to kCounterInts of them (so that a workspace reused across shapes keeps
// them at zero: the partials never land there), then the splits' partials.
constexpr size_t kCounterInts = TRA_NOALLOC_MAX_COUNTERS;
size_t decode_counter_bytes(int32_t B, int32_t Hkv) {
  const size_t n = (size_t)B * (Hkv + 1);
  return round256(4 * (n > kCounterInts ? n : kCounterInts));
}

size_t tra_decode_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t d) {
  if (B < 1 || Hq < 1 || Hkv < 1 || d < 1) return 0;
  const size_t S = (size_t)tra::decode_splits(B, Hkv);
  return decode_counter_bytes(B, Hkv) + round256((size_t)B * Hq * S * 2 * 4) +
         round256((size_t)B * Hq * S * d * 4);
}

tra_status routed_attention_decode(const tra_shape* shape, const tra_policy* policy,
                                   const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                                   const tra_qtiles* cache, const int32_t* row_ptr,
                                   const uint32_t* entries, uint16_t* k_tail, uint16_t* v_tail,
                                   int32_t* tail_len_dev, int32_t tail_cap, float softmax_scale,
                                   uint16_t* out, void* workspace, size_t workspace_bytes,
                                   int32_t* status_dev, void* stream) {
  const CallRange range("tra::routed_attention_decode");
  int64_t nt = 0, ntok = 0, nt_max = 0;
  tra_status st = check_shape(shape, &nt, &ntok, &nt_max);
  if (st != TRA_OK) return st;
  st = check_policy(shape, policy, nt_max);
  if (st != TRA_OK) return st;
  if (shape->Hq / shape->Hkv > 8) return fail(TRA_ERR_UNSUPPORTED, "decode supports Hq/Hkv <= 8");
  if (!q || !k_new || !v_new || !cache || !row_ptr || !entries || !k_tail || !v_tail ||
      !tail_len_dev || !out || !workspace || !status_dev)
    return fail(TRA_ERR_INVALID, "a required pointer is NULL");
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_tail) ||
      !aligned16(v_tail) || !aligned16(out) || !aligned16(workspace))
    return fail(TRA_ERR_INVALID, "q/k_new/v_new/tails/out/workspace must be 16-byte aligned");
  if (tail_cap < 1) return fail(TRA_ERR_INVALID, "tail_cap must be >= 1");
  const uint32_t need8 = TRA_FMT_K8 | TRA_FMT_V8;
  if ((cache->formats & need8) != need8 || !cache->k8 || !cache->v8 || !cache->sk8 || !cache->sv8)
    return fail(TRA_ERR_INVALID, "decode needs K8 and V8 cache tiles");
  if (!aligned16(cache->k8) || !aligned16(cache->v8)) return fail(TRA_ERR_INVALID, "K8/V8 misaligned");
  if (policy_has_int4(shape, policy)) {
    const uint32_t need4 = TRA_FMT_K4 | TRA_FMT_V4;
    if ((cache->formats & need4) != need4 || !cache->k4 || !cache->v4 || !cache->sk4 || !cache->sv4)
      return fail(TRA_ERR_INVALID, "the policy has INT4 tiles: K4 and V4 cache tiles are required");
    if (!aligned16(cache->k4) || !aligned16(cache->v4)) return fail(TRA_ERR_INVALID, "K4/V4 misaligned");
  }
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale))
    return fail(TRA_ERR_INVALID, "softmax_scale must be positive and finite");
  const size_t need = tra_decode_workspace_bytes(shape->B, shape->Hq, shape->Hkv, shape->d);
  if (workspace_bytes < need) return fail(TRA_ERR_BUFFER, "workspace needs %zu bytes", need);
  tra::DecodeParams p{};
  p.cu = shape->cu_seqlens_dev;
  p.B = shape->B;
  p.Hq = shape->Hq;
  p.Hkv = shape->Hkv;
  p.d = shape->d;
  p.ntiles = (int)nt;
  p.splits = tra::decode_splits(shape->B, shape->Hkv);
  p.q = q;
  p.k_new = k_new;
  p.v_new = v_new;
  p.sk8 = cache->sk8;
  p.sk4 = cache->sk4;
  p.sv8 = cache->sv8;
  p.sv4 = cache->sv4;
  p.row_ptr = row_ptr;
  p.entries = entries;
  p.k_tail = k_tail;
  p.v_tail = v_tail;
  p.tail_len = tail_len_dev;
  p.tail_cap = tail_cap;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out;
  const size_t S = (size_t)p.splits;
  uint8_t* const ws = reinterpret_cast<uint8_t*>(workspace);
  p.row_count = reinterpret_cast<int32_t*>(ws);
  p.seq_count = p.row_count + (size_t)shape->B * shape->Hkv;
  const size_t off_ml = decode_counter_bytes(shape->B, shape->Hkv);
  p.part_ml = reinterpret_cast<float*>(ws + off_ml);
  p.part_o = reinterpret_cast<float*>(ws + off_ml + round256((size_t)shape->B * shape->Hq * S * 2 * 4));
  p.status = status_dev;
  tra::DecodeMaps m;
  memset(&m, 0, sizeof m);
  const int64_t rows = (int64_t)shape->Hkv * nt * TRA_TILE;
  const bool has4 = cache->k4 && cache->v4;  // INT4 maps unused (never loaded) without INT4 tiles
  bool good = map_i8(&m.k8, cache->k8, shape->d, rows, 64) &&
              map_i8(&m.v8, cache->v8, shape->d, rows, 64) &&
              map_i8(&m.k4, has4 ? (const void*)cache->k4 : cache->k8, shape->d / 2, rows, 64) &&
              map_i8(&m.v4, has4 ? (const void*)cache->v4 : cache->v8, shape->d / 2, rows, 64);
  if (!good) return fail(TRA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  cudaError_t e = tra::launch_decode(p, m, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return ok();
}

int32_t tra_hybrid_capacity(const tra_shape* shape, double frac) {
  if (check_shape(shape, nullptr, nullptr, nullptr) != TRA_OK) return -1;
  if (!(frac >= 0.0 && frac <= 1.0)) return -1;
  int64_t m = 0;
  for (int b = 0; b < shape->B; ++b) {
    const int64_t T = (int64_t)shape->cu_seqlens_host[b + 1] - shape->cu_seqlens_host[b];
    const int64_t n = std::min<int64_t>(T, (int64_t)std::ceil(frac * (double)T));
    m = std::max(m, n);
  }
  return (int32_t)m;
}

static tra_status check_hybrid(const tra_shape* shape, const tra_hybrid* hy, int64_t nt) {
  if (!hy) return fail(TRA_ERR_INVALID, "hybrid arrays are NULL");
  if (hy->window < 0) return fail(TRA_ERR_INVALID, "window must be >= 0 (got %d)", hy->window);
  if (hy->cap < 0) return fail(TRA_ERR_INVALID, "cap must be >= 0");
  if (!hy->sel_count || !hy->sel_pos || !hy->sel_mask || (hy->cap > 0 && (!hy->k_sel || !hy->v_sel)) ||
      (hy->window > 0 && (!hy->k_win || !hy->v_win)))
    return fail(TRA_ERR_INVALID, "a hybrid array is NULL");
  if (!aligned16(hy->sel_mask) || !aligned16(hy->sel_pos) || (hy->k_sel && !aligned16(hy->k_sel)) ||
      (hy->v_sel && !aligned16(hy->v_sel)) || (hy->k_win && !aligned16(hy->k_win)) ||
      (hy->v_win && !aligned16(hy->v_win)))
    return fail(TRA_ERR_INVALID, "hybrid arrays must be 16-byte aligned");
  (void)shape;
  (void)nt;
  return TRA_OK;
}

tra_status hybrid_select_tokens(const tra_shape* shape, const float* importance, double frac,
                                const uint16_t* k, const uint16_t* v, const tra_hybrid* hy,
                                void* stream) {
  const CallRange range("tra::hybrid_select_tokens");
  int64_t nt = 0, ntok = 0;
  tra_status st = check_shape(shape, &nt, &ntok, nullptr);
  if (st != TRA_OK) return st;
  if (!(frac >= 0.0 && frac <= 1.0)) return fail(TRA_ERR_INVALID, "frac must lie in [0, 1]");
  if (!importance || !k || !v) return fail(TRA_ERR_INVALID, "importance, k and v are required");
  if (!aligned16(k) || !aligned16(v) || (reinterpret_cast<uintptr_t>(importance) & 3u))
    return fail(TRA_ERR_INVALID, "k / v must be 16-byte aligned, importance 4-byte aligned");
  st = check_hybrid(shape, hy, nt);
  if (st != TRA_OK) return st;
  const int32_t need = tra_hybrid_capacity(shape, frac);
  if (hy->cap < need) return fail(TRA_ERR_BUFFER, "cap %d < %d selected tokens", hy->cap, need);
  if (nt == 0) return ok();
  tra::HybridSelectParams p{};
  p.cu = shape->cu_seqlens_dev;
  p.B = shape->B;
  p.Hkv = shape->Hkv;
  p.d = shape->d;
  p.ntiles = (int)nt;
  p.cap = hy->cap;
  p.window = hy->window;
  p.frac = frac;
  p.imp = importance;
  p.k = k;
  p.v = v;
  p.sel_count = hy->sel_count;
  p.sel_pos = hy->sel_pos;
  p.sel_mask = hy->sel_mask;
  p.k_sel = hy->k_sel;
  p.v_sel = hy->v_sel;
  p.k_win = hy->k_win;
  p.v_win = hy->v_win;
  cudaError_t e = tra::launch_hybrid_select(p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hybrid select launch");
  return ok();
}

tra_status hybrid_attention_decode(const tra_shape* shape, const tra_hybrid* hy, const uint16_t* q,
                                   const uint16_t* k_new, const uint16_t* v_new,
                                   const tra_qtiles* cache, uint16_t* k_tail, uint16_t* v_tail,
                                   int32_t* tail_len_dev, int32_t tail_cap, float softmax_scale,
                                   uint16_t* out, void* workspace, size_t workspace_bytes,
                                   int32_t* status_dev, void* stream) {
  const CallRange range("tra::hybrid_attention_decode");
  int64_t nt = 0, ntok = 0, nt_max = 0;
  tra_status st = check_shape(shape, &nt, &ntok, &nt_max);
  if (st != TRA_OK) return st;
  st = check_hybrid(shape, hy, nt);
  if (st != TRA_OK) return st;
  if (shape->Hq / shape->Hkv > 8) return fail(TRA_ERR_UNSUPPORTED, "decode supports Hq/Hkv <= 8");
  if (!q || !k_new || !v_new || !cache || !k_tail || !v_tail || !tail_len_dev || !out || !workspace ||
      !status_dev)
    return fail(TRA_ERR_INVALID, "a required pointer is NULL");
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_tail) ||
      !aligned16(v_tail) || !aligned16(out) || !aligned16(workspace))
    return fail(TRA_ERR_INVALID, "q/k_new/v_new/tails/out/workspace must be 16-byte aligned");
  if (tail_cap < 1) return fail(TRA_ERR_INVALID, "tail_cap must be >= 1");
  const uint32_t need4 = TRA_FMT_K4 | TRA_FMT_V4;
  if ((cache->formats & need4) != need4 || !cache->k4 || !cache->v4 || !cache->sk4 || !cache->sv4)
    return fail(TRA_ERR_INVALID, "the hybrid decode reads K4 and V4 cache tiles");
  if (!aligned16(cache->k4) || !aligned16(cache->v4)) return fail(TRA_ERR_INVALID, "K4/V4 misaligned");
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale))
    return fail(TRA_ERR_INVALID, "softmax_scale must be positive and finite");
  const size_t need = tra_decode_workspace_bytes(shape->B, shape->Hq, shape->Hkv, shape->d);
  if (workspace_bytes < need) return fail(TRA_ERR_BUFFER, "workspace needs %zu bytes", need);
  tra::DecodeParams p{};
  p.cu = shape->cu_seqlens_dev;
  p.B = shape->B;
  p.Hq = shape->Hq;
  p.Hkv = shape->Hkv;
  p.d = shape->d;
  p.ntiles = (int)nt;
  p.splits = tra::decode_splits(shape->B, shape->Hkv);
  p.q = q;
  p.k_new = k_new;
  p.v_new = v_new;
  p.sk4 = cache->sk4;
  p.sv4 = cache->sv4;
  p.k_tail = k_tail;
  p.v_tail = v_tail;
  p.tail_len = tail_len_dev;
  p.tail_cap = tail_cap;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out;
  const size_t S = (size_t)p.splits;
  uint8_t* const ws = reinterpret_cast<uint8_t*>(workspace);
  p.row_count = reinterpret_cast<int32_t*>(ws);
  p.seq_count = p.row_count + (size_t)shape->B * shape->Hkv;
  const size_t off_ml = decode_counter_bytes(shape->B, shape->Hkv);
  p.part_ml = reinterpret_cast<float*>(ws + off_ml);
  p.part_o = reinterpret_cast<float*>(ws + off_ml + round256((size_t)shape->B * shape->Hq * S * 2 * 4));
  p.status = status_dev;
  p.sel_count = hy->sel_count;
  p.sel_mask = hy->sel_mask;
  p.k_sel = hy->k_sel;
  p.v_sel = hy->v_sel;
  p.k_win = hy->k_win;
  p.v_win = hy->v_win;
  p.sel_cap = hy->cap;
  p.window = hy->window;
  tra::DecodeMaps m;
  memset(&m, 0, sizeof m);
  const int64_t rows = (int64_t)shape->Hkv * nt * TRA_TILE;
  bool good = map_i8(&m.k4, cache->k4, shape->d / 2, rows, 64) &&
              map_i8(&m.v4, cache->v4, shape->d / 2, rows, 64);
  m.k8 = m.k4;  // (INT8 maps unused: every prefix tile is read in INT4)
  m.v8 = m.v4;
  if (!good) return fail(TRA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  cudaError_t e = tra::launch_decode(p, m, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "hybrid decode launch");
  return ok();
}

tra_status hybrid_attention_prefill(const tra_shape* shape, const tra_hybrid* hy, const uint16_t* q,
                                    const uint16_t* k, const uint16_t* v, const tra_qtiles* kv,
                                    uint16_t* k_mix, uint16_t* v_mix, float softmax_scale,
                                    uint16_t* out, float* lse, int32_t* status_dev, void* stream) {
  const CallRange range("tra::hybrid_attention_prefill");
  int64_t nt = 0, ntok = 0, nt_max = 0;
  tra_status st = check_shape(shape, &nt, &ntok, &nt_max);
  if (st != TRA_OK) return st;
  if (!hy || !hy->sel_mask) return fail(TRA_ERR_INVALID, "the hybrid selection masks are required");
  if (hy->window < 0) return fail(TRA_ERR_INVALID, "window must be >= 0 (got %d)", hy->window);
  if (!q || !k || !v || !kv || !k_mix || !v_mix || !out || !status_dev)
    return fail(TRA_ERR_INVALID, "q, k, v, kv, k_mix, v_mix, out and status are required");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(k_mix) || !aligned16(v_mix) ||
      !aligned16(out) || !aligned16(hy->sel_mask) || (lse && !aligned16(lse)))
    return fail(TRA_ERR_INVALID, "q/k/v/k_mix/v_mix/out/lse/sel_mask must be 16-byte aligned");
  if (!(kv->formats & (TRA_FMT_K4 | TRA_FMT_K4X)) || !(kv->formats & TRA_FMT_V4) || !kv->sk4 ||
      !kv->sv4)
    return fail(TRA_ERR_INVALID, "the hybrid prefill needs the K and V INT4 tile scales (K4 or K4X, V4)");
  if (nt_max >= (1ll << 24)) return fail(TRA_ERR_UNSUPPORTED, "a sequence has more than 2^24 tiles");
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale))
    return fail(TRA_ERR_INVALID, "softmax_scale must be positive and finite");
  if (ntok == 0 || nt == 0) return ok();
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  tra::HybridMixParams mp{};
  mp.cu = shape->cu_seqlens_dev;
  mp.B = shape->B;
  mp.Hkv = shape->Hkv;
  mp.d = shape->d;
  mp.ntiles = (int)nt;
  mp.k = k;
  mp.v = v;
  mp.sk4 = kv->sk4;
  mp.sv4 = kv->sv4;
  mp.sel_mask = hy->sel_mask;
  mp.k_mix = k_mix;
  mp.v_mix = v_mix;
  cudaError_t e = tra::launch_hybrid_mix(mp, s);
  if (e != cudaSuccess) return cuda_fail(e, "hybrid mix launch");
  tra::PrefillParams p{};
  p.cu = shape->cu_seqlens_dev;
  p.B = shape->B;
  p.Hq = shape->Hq;
  p.Hkv = shape->Hkv;
  p.d = shape->d;
  p.ntiles = (int)nt;
  p.mode = tra::kPrefillModeHybrid;
  p.jmax = (int)((nt_max + 1) / 2);
  p.sk4 = kv->sk4;
  p.sv4 = kv->sv4;
  p.sel_mask = hy->sel_mask;
  p.window = hy->window;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out;
  p.lse = lse;
  p.status = status_dev;
  tra::PrefillMaps m;
  memset(&m, 0, sizeof m);
  const int d = shape->d;
  bool good = map_bf16(&m.qb, q, d, shape->Hq, ntok, 128) &&
              map_bf16(&m.kb, k, d, shape->Hkv, ntok, 64) &&
              map_bf16(&m.vb, v, d, shape->Hkv, ntok, 64) &&
              map_bf16(&m.kmix, k_mix, d, shape->Hkv, ntok, 64) &&
              map_bf16(&m.vmix, v_mix, d, shape->Hkv, ntok, 64);
  if (!good) return fail(TRA_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  e = tra::launch_prefill(p, m, s);
  if (e != cudaSuccess) return cuda_fail(e, "hybrid prefill launch");
  return ok();
}

tra_status tra_boundary_tile_counts(const tra_shape* shape, int32_t b1, int32_t b2, int64_t* n8,
                                    int64_t* n4) {
  tra_status st = check_shape(shape, nullptr, nullptr, nullptr);
  if (st != TRA_OK) return st;
  if (!n8 || !n4) return fail(TRA_ERR_INVALID, "n8/n4 outputs are NULL");
  if (b1 < 1 || b2 < b1) return fail(TRA_ERR_INVALID, "need 1 <= b1 <= b2 (got %d, %d)", b1, b2);
  const int32_t* cu = shape->cu_seqlens_host;
  int64_t kept8 = 0, kept = 0;
  for (int b = 0; b < shape->B; ++b) {
    const int64_t n = ceil_tiles(cu[b + 1] - cu[b]);
    kept8 += tri_capped(n, b1);
    kept += tri_capped(n, b2);
  }
  *n8 = kept8;
  *n4 = kept - kept8;
  return ok();
}

tra_status tra_prefill_cost_model(const tra_shape* shape, const int32_t* b1, const int32_t* b2,
                                  double dual_weight, double solo, int32_t n_sm, double* makespan,
                                  double* entries) {
  int64_t nt = 0, nt_max = 0;
  tra_status st = check_shape(shape, &nt, nullptr, &nt_max);
  if (st != TRA_OK) return st;
  tra_policy pol{};
  pol.mode = TRA_POLICY_BOUNDARY;
  pol.b1 = b1;
  pol.b2 = b2;
  st = check_policy(shape, &pol, nt_max);
  if (st != TRA_OK) return st;
  if (!(dual_weight >= 1.0) || !(solo > 0.0 && solo <= 1.0) || n_sm < 1 || !makespan || !entries)
    return fail(TRA_ERR_INVALID, "need dual_weight >= 1, 0 < solo <= 1, n_sm >= 1 and outputs");
  const int32_t* cu = shape->cu_seqlens_host;
  const int Hq = shape->Hq, B = shape->B;
  const int64_t jmax = (nt_max + 1) / 2;
  // precision a q-tile row gives k-tile kt under (b1, b2): 2 INT8, 1 INT4, 0 skipped
  auto prec = [](int64_t qt, int64_t kt, int32_t lo1, int32_t lo2) -> int {
    if (kt > qt || kt < 0) return 0;
    const int64_t dist = qt - kt;
    return dist < lo1 ? 2 : (dist < lo2 ? 1 : 0);
  };
  // work of unit id (launch order: q-tile pairs from the heaviest, then sequence, then head)
  auto unit_work = [&](int64_t id, double* cnt) -> double {
    const int h = (int)(id % Hq);
    const int b = (int)((id / Hq) % B);
    const int64_t j = jmax - 1 - id / ((int64_t)Hq * B);
    const int64_t ntb = ceil_tiles(cu[b + 1] - cu[b]);
    const int64_t q0 = 2 * j, q1 = 2 * j + 1;
    if (q0 >= ntb) return 0.0;
    const bool second = q1 < ntb;
    double w = 0.0;
    const int64_t lo = std::max<int64_t>(0, q0 - b2[h] + 1);
    const int64_t hi = second ? q1 : q0;
    for (int64_t kt = lo; kt <= hi; ++kt) {
      const int pa = prec(q0, kt, b1[h], b2[h]);
      const int pb = second ? prec(q1, kt, b1[h], b2[h]) : 0;
      if (!pa && !pb) continue;
      w += (pa && pb && pa != pb) ? dual_weight : 1.0;
      *cnt += 1.0;
    }
    return w;
  };
  const int64_t units = jmax * B * Hq;
  const int64_t ctas = (units + 1) / 2;
  std::vector<double> sm((size_t)n_sm, 0.0);  // time each SM frees up
  double total = 0.0;
  for (int64_t c = 0; c < ctas; ++c) {
    const double w0 = unit_work(2 * c, &total), w1 = unit_work(2 * c + 1, &total);
    const double w = std::min(w0, w1) + solo * std::fabs(w0 - w1);
    if (w == 0.0) continue;  // an empty CTA exits at once
    auto it = std::min_element(sm.begin(), sm.end());
    *it += w;
  }
  *makespan = *std::max_element(sm.begin(), sm.end());
  *entries = total;
  return ok();
}

tra_status tra_allocate_boundaries(int32_t n_heads, int32_t n_cand, const double* err,
                                   const int64_t* cost, int64_t budget, int32_t* choice,
                                   double* total_err, int64_t* total_cost) {
  if (n_heads < 1 || n_cand < 1 || n_cand > 255)
    return fail(TRA_ERR_INVALID, "need n_heads >= 1 and 1 <= n_cand <= 255 (got %d, %d)", n_heads, n_cand);
  if (!err || !cost || !choice) return fail(TRA_ERR_INVALID, "err, cost and choice are required");
  if (budget < 0) return fail(TRA_ERR_INVALID, "budget < 0");
  if ((double)n_heads * ((double)budget + 1.0) > (double)(1ll << 27))
    return fail(TRA_ERR_UNSUPPORTED, "n_heads x (budget + 1) = %.0f exceeds 2^27: use coarser cost units",
                (double)n_heads * ((double)budget + 1.0));
  const size_t nh = (size_t)n_heads, nc = (size_t)n_cand, nb = (size_t)budget + 1;
  for (size_t i = 0; i < nh * nc; ++i) {
    if (!std::isfinite(err[i])) return fail(TRA_ERR_INVALID, "err[%zu] is not finite", i);
    if (cost[i] < 0) return fail(TRA_ERR_INVALID, "cost[%zu] < 0", i);
  }
  // per head, the candidates no other one beats on both cost and error, by rising cost
  std::vector<std::vector<int>> front(nh);
  for (size_t h = 0; h < nh; ++h) {
    std::vector<int> idx(nc);
    for (size_t c = 0; c < nc; ++c) idx[c] = (int)c;
    const double* e = err + h * nc;
    const int64_t* k = cost + h * nc;
    std::sort(idx.begin(), idx.end(), [&](int a, int b) {
      if (k[a] != k[b]) return k[a] < k[b];
      if (e[a] != e[b]) return e[a] < e[b];
      return a < b;
    });
    double best = INFINITY;
    for (int c : idx)
      if (e[c] < best && k[c] <= budget) {
        front[h].push_back(c);
        best = e[c];
      }
    if (front[h].empty())
      return fail(TRA_ERR_INVALID, "head %zu has no candidate within the budget", h);
  }
  // f[B]: least total error of the heads so far with total cost <= B
  std::vector<double> f(nb, 0.0), g(nb);
  std::vector<uint8_t> pick(nh * nb);
  for (size_t h = 0; h < nh; ++h) {
    const double* e = err + h * nc;
    const int64_t* k = cost + h * nc;
    for (size_t B = 0; B < nb; ++B) {
      double v = INFINITY;
      uint8_t pk = 0;
      for (size_t j = 0; j < front[h].size(); ++j) {
        const int c = front[h][j];
        if ((size_t)k[c] > B) break;  // the front rises in cost
        const double t = e[c] + f[B - (size_t)k[c]];
        if (t < v) {
          v = t;
          pk = (uint8_t)j;
        }
      }
      g[B] = v;
      pick[h * nb + B] = pk;
    }
    f.swap(g);
  }
  if (!(f[nb - 1] < INFINITY)) return fail(TRA_ERR_INVALID, "no choice of candidates fits the budget");
  size_t B = nb - 1;
  int64_t spent = 0;
  for (size_t h = nh; h-- > 0;) {
    const int c = front[h][pick[h * nb + B]];
    choice[h] = c;
    B -= (size_t)cost[h * nc + c];
    spent += cost[h * nc + c];
  }
  if (total_err) *total_err = f[nb - 1];
  if (total_cost) *total_cost = spent;
  return ok();
}

tra_status tra_selftest_bounded_wait(int32_t* status_dev, int64_t limit_ns, void* stream) {
  if (!status_dev) return fail(TRA_ERR_INVALID, "status_dev is NULL");
  if (limit_ns < 1000 || limit_ns > 1000000000)
    return fail(TRA_ERR_INVALID, "limit_ns must lie in [1e3, 1e9] (got %lld)", (long long)limit_ns);
  cudaError_t e = tra::launch_wait_selftest(status_dev, (uint64_t)limit_ns,
                                            reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return ok();
}

}  // extern "C"
