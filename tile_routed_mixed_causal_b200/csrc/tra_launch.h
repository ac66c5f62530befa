// tra_launch.h -- internal launch parameter blocks shared by the host ABI
// (tra_api.cu) and the kernel files.  Not part of the public C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tra.h"

namespace tra {

// ------------------------------------------------------------ quantisation
struct QuantTensor {
  const uint16_t* x;   // bf16 [ntok][H][d]
  int H;
  int8_t* x8;          // nullable
  uint8_t* x4;         // nullable
  int8_t* x4x;         // nullable: INT4 codes as int8 values 16 x code, row-major
  float* s8;
  float* s4;
  int perm4;           // x4 in the decode's V fragment order (V), else row-major
  int bias8;           // x8 codes stored offset-binary, code + 128 (V), else two's complement
  uint8_t* xf;         // nullable: FP8 E4M3 codes, row-major
  float* sf;           // their scales
};

struct QuantParams {
  QuantTensor t[3];          // Q, K, V (H = 0 or x = null: skipped)
  long long cta_begin[4];    // prefix of H*ntiles over the three tensors
  const int32_t* cu;         // device cu_seqlens
  int B, d, ntiles;
};

cudaError_t launch_quantize(const QuantParams& p, cudaStream_t s);

// ------------------------------------------------------------ traversal lists
struct ListParams {
  const int32_t* cu;
  int B, Hq, Hkv, ntiles, mode, kind;
  const uint32_t* bitmask;
  int G, W;
  int32_t* row_ptr;
  uint32_t* entries;
  long long rows;
  int32_t b1[TRA_MAX_HEADS];
  int32_t b2[TRA_MAX_HEADS];
  int32_t b8[TRA_MAX_HEADS];  // FP8 band [b1, b8) of a boundary policy (b8 = b1: none)
};

cudaError_t launch_lists(const ListParams& p, cudaStream_t s);

// ------------------------------------------------------------ prefill
struct PrefillParams {
  const int32_t* cu;
  int B, Hq, Hkv, d, ntiles;
  int mode;              // TRA_POLICY_*
  int has_int4;          // Q4X/K4X tiles present (boundary policies with some b1 < b2)
  int jmax;              // max over sequences of ceil(nt/2) (q-tile pairs)
  const int32_t* row_ptr;
  const uint32_t* entries;
  const float* sq8;
  const float* sq4;
  const float* sk8;
  const float* sk4;
  float scale_log2;      // softmax_scale * log2(e)
  uint16_t* out;         // bf16 [ntok][Hq][d]
  float* lse;            // [Hq][ntok] or null
  const int32_t* dump_coords;
  int n_dump;
  int32_t* dump_out;
  int32_t* status;
  // token-level hybrid prefill (mode kPrefillModeHybrid): INT4 scales of V, the
  // per-tile selection masks [Hkv][ntiles] and the window (keys closer than it to
  // the query are read in bf16)
  const float* sv4;
  const uint64_t* sel_mask;
  int window;
  // FP8 band (mode kPrefillModeBoundaryF8): scales of the E4M3 Q and K tiles
  const float* sqf;
  const float* skf;
  // boundary policies: b1 and b8 (b8 = b1 without an FP8 band) per query head, which fix
  // the lengths of a traversal row's precision runs
  int32_t b1[TRA_MAX_HEADS];
  int32_t b8[TRA_MAX_HEADS];
};

// prefill modes beside the TRA_POLICY_* ones: the token-level hybrid, and a boundary
// policy with an FP8 band
constexpr int kPrefillModeHybrid = 3;
constexpr int kPrefillModeBoundaryF8 = 4;

struct PrefillMaps {
  CUtensorMap q8, k8;    // int8 tiles, 2-D (d bytes x rows)
  CUtensorMap q4x, k4x;  // expanded INT4 tiles (int8 16 x code), 2-D like q8 / k8
  CUtensorMap qb, kb, vb;  // bf16, 3-D (d, H, ntok)
  CUtensorMap kmix, vmix;  // hybrid: mixed K / V operands, bf16 3-D like kb / vb
  CUtensorMap qf8, kf8;    // FP8 E4M3 tiles, 2-D like q8 / k8
};

cudaError_t launch_prefill(const PrefillParams& p, const PrefillMaps& m, cudaStream_t s);

// ------------------------------------------------------------ decode
struct DecodeParams {
  const int32_t* cu;
  int B, Hq, Hkv, d, ntiles, splits;
  const uint16_t* q;       // [B][Hq][d]
  const uint16_t* k_new;   // [B][Hkv][d]
  const uint16_t* v_new;
  const float* sk8;
  const float* sk4;
  const float* sv8;
  const float* sv4;
  const int32_t* row_ptr;
  const uint32_t* entries;
  uint16_t* k_tail;        // [B][Hkv][cap][d]
  uint16_t* v_tail;
  int32_t* tail_len;
  int tail_cap;
  float scale_log2;
  uint16_t* out;           // [B][Hq][d]
  float* part_ml;          // [B][Hq][splits][2]
  float* part_o;           // [B][Hq][splits][d]
  int32_t* row_count;      // [B][Hkv] splits finished this step (zero between calls)
  int32_t* seq_count;      // [B] rows finished this step (zero between calls)
  int32_t* status;
  // token-level hybrid (hybrid_attention_decode; null otherwise): every prefix tile is
  // read in INT4 except its selected / in-window keys, which come from the bf16 side
  const int32_t* sel_count;
  const uint64_t* sel_mask;
  const uint16_t* k_sel;
  const uint16_t* v_sel;
  const uint16_t* k_win;
  const uint16_t* v_win;
  int sel_cap, window;
};

struct DecodeMaps {
  CUtensorMap k8, v8;      // int8 codes, 2-D (d bytes x rows), box 64 rows
  CUtensorMap k4, v4;      // packed INT4 codes (d/2 bytes x rows)
};

// ------------------------------------------------------------ token-level hybrid
struct HybridSelectParams {
  const int32_t* cu;
  int B, Hkv, d, ntiles, cap, window;
  double frac;
  const float* imp;        // [ntok][Hkv]
  const uint16_t* k;       // [ntok][Hkv][d] bf16
  const uint16_t* v;
  int32_t* sel_count;      // [B]
  int32_t* sel_pos;        // [B][Hkv][cap]
  uint64_t* sel_mask;      // [Hkv][ntiles]
  uint16_t* k_sel;         // [B][Hkv][cap][d]
  uint16_t* v_sel;
  uint16_t* k_win;         // [B][Hkv][window][d]
  uint16_t* v_win;
};

cudaError_t launch_hybrid_select(const HybridSelectParams& p, cudaStream_t s);

// Mixed K / V operands of the hybrid prefill: each key row is the token's bf16 row
// when its tile's selection mask marks it, else its INT4 codes (the tile's INT4
// scale, as the quantiser computes them) written as bf16 integers.
struct HybridMixParams {
  const int32_t* cu;
  int B, Hkv, d, ntiles;
  const uint16_t* k;         // [ntok][Hkv][d] bf16
  const uint16_t* v;
  const float* sk4;          // [Hkv][ntiles]
  const float* sv4;
  const uint64_t* sel_mask;  // [Hkv][ntiles]
  uint16_t* k_mix;           // [ntok][Hkv][d] bf16
  uint16_t* v_mix;
};

cudaError_t launch_hybrid_mix(const HybridMixParams& p, cudaStream_t s);

int decode_splits(int B, int Hkv);
cudaError_t launch_wait_selftest(int32_t* status, uint64_t limit_ns, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams& p, const DecodeMaps& m, cudaStream_t s);

// Records `msg` as this thread's tra_last_error() text and returns `st`.
tra_status report_error(tra_status st, const char* msg);

}  // namespace tra
