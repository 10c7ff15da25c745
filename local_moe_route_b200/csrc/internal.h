// internal.h -- launchers shared between the C-ABI layer (api.cu) and the
// kernel translation units.  Host-side only declarations; no torch types.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace strata {

// Tile of token rows handled by one tcgen05 GEMM work unit.
constexpr int kTileRows = 160;
// Token slots per histogram chunk in the permutation.
constexpr int kPermChunk = 1024;
// Batches of at most this many tokens use the weight-streaming expert kernel.
constexpr int kStreamMaxTokens = 8;

// Per-expert work lists derived from offsets (built on the device).
struct Schedule {
  int32_t* tile_prefix;   // [E+1]  tiles before expert e; [E] = total
  int4* tile_table;       // [max_tiles] (expert, first grouped row, rows, 0)
  int32_t* active;        // [E]   experts with at least one row, ascending
  int32_t* n_active;      // [1]
};

inline int max_tiles(int S, int E) {
  return S / kTileRows + (S < E ? S : E) + 1;
}

// Streaming multiprocessors of the current device (looked up once per device).
int sm_count();

// Resolves a driver entry point once (the tensor-map encoder).
CUresult encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                        uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                        uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle,
                        CUtensorMapL2promotion promo);

// ---- routing
cudaError_t launch_router_logits_tc(const uint16_t* x, const uint16_t* w_router, int T, int d,
                                    int E, float* logits, unsigned* err, cudaStream_t s);
cudaError_t launch_router_logits_simt(const uint16_t* x, const uint16_t* w_router, int T, int d,
                                      int E, int ksplit, float* partial, cudaStream_t s);
cudaError_t launch_topk_softmax(const float* partial, int ksplit, const float* bias, int T,
                                int E, int k, int32_t* ids, float* w, float* logits_out,
                                cudaStream_t s);
bool router_uses_tc(int T, int d, int E);
int router_ksplit(int T, int d, int E);

// ---- grouping
cudaError_t launch_permute(const int32_t* ids, int T, int k, int E, int32_t* counts,
                           int32_t* offsets, int32_t* sorted_token, int32_t* slot_row,
                           int32_t* hist, unsigned* err, cudaStream_t s);
// tile_rows: token rows per tile of the tensor-core GEMM that follows
// (kTileRows); max_tiles bounds the table for tiles of at least kTileRows.
cudaError_t launch_schedule(const int32_t* offsets, int E, int S, int tile_rows, Schedule sch,
                            unsigned* err, cudaStream_t s);

// ---- expert GEMMs
struct GemmProblem {
  int op;                       // 0 gate/up + SwiGLU, 1 down
  const uint16_t* a;            // x [T][d] or h [S][n]
  const int32_t* sorted_token;  // gate/up only
  const int32_t* offsets;       // [E+1]
  const uint8_t* q0; const uint16_t* s0;  // gate (or down)
  const uint8_t* q1; const uint16_t* s1;  // up (gate/up only)
  const float* row_scale;       // down only, nullable
  uint16_t* a16;                // scratch [T*k][d]: fp16 x rows in grouped order (TC gate/up)
  uint16_t* out;
  int T, S, E, K, N, G;         // K reduction dim, N output features
  // Tensor-core path only, set by the fused forward: h travels between the
  // two GEMMs with its features interleaved within groups of 8 (0,4,1,5,
  // 2,6,3,7), the order the down projection's weight dequantisation
  // produces: gate/up writes it that way, down reads it that way.
  bool h_interleaved = false;
  unsigned* err;
};
cudaError_t launch_gemm_tc(const GemmProblem& p, const Schedule& sch, cudaStream_t s);
// Gate/up B operand: xs[p] = fp16(x[sorted_token[p]]), features interleaved
// within groups of 8 (0, 4, 1, 5, 2, 6, 3, 7).
cudaError_t launch_gather_rows_f16(const uint16_t* x, const int32_t* sorted_token, int T, int d,
                                   int S, uint16_t* xs, unsigned* err, cudaStream_t s);
cudaError_t launch_gemm_stream(const GemmProblem& p, const Schedule& sch, cudaStream_t s);
// Decode batches with K % 256 == 0, N % 64 == 0 and a group of 32, 64 or 128
// (weights staged by TMA); cudaErrorNotSupported for other shapes.
cudaError_t launch_gemm_decode(const GemmProblem& p, const Schedule& sch, cudaStream_t s);

// ---- the whole layer for batches of at most four tokens, one launch
bool decode_fused_fits(int T, int d, int E, int k, int n, int G);
size_t decode_fused_scratch(int T, int d, int E, int k, int n);
cudaError_t launch_decode_fused(const uint16_t* x, const uint16_t* w_router, const float* bias,
                                const uint8_t* q_gate, const uint16_t* s_gate,
                                const uint8_t* q_up, const uint16_t* s_up,
                                const uint8_t* q_down, const uint16_t* s_down, int T, int d,
                                int E, int k, int n, int G, uint16_t* y, int32_t* ids_out,
                                float* w_out, void* scratch, unsigned* err, cudaStream_t s);

// ---- combine
cudaError_t launch_combine_checked(const uint16_t* rows, const float* w, const int32_t* slot_row,
                                   int T, int k, int d, uint16_t* y, unsigned* err,
                                   cudaStream_t s);

cudaError_t launch_gather_rows(const uint16_t* src, const int32_t* index, int src_rows,
                               int rows, int width, uint16_t* dst, unsigned* err,
                               cudaStream_t s);

// ---- attention over indexer-selected KV rows
size_t sparse_attn_scratch(int T, int Hq, int P, int D);
cudaError_t launch_sparse_attn(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                               const int32_t* idx, int T, int L, int Hq, int Hkv, int D, int P,
                               float scale, uint16_t* out, void* ws, unsigned* err,
                               cudaStream_t s);

}  // namespace strata
