// The surrounding Swimba block and its causal convolution: C ABI entry points.
//
// Block ("Mamba y las SSMs: el retorno del estado persistente", section "Mamba", Figura 3, and
// section "Estado interno puramente lineal"; "Swimba: Switch Mamba Model Scales State Space
// Models", Dutch summary §2 "Architectuur Implementatie"):
//   [x_pre | z] = u W_in;  x = SiLU(causal depthwise conv(x_pre));  the Swimba layer on (x, z);
//   o = layer_out W_out + u.
// The two projections are dense GEMMs on the library's own kernel (gemm.cu: tcgen05 for bf16,
// SIMT for fp32): the in-projection's epilogue splits its columns into x_pre and z, the
// out-projection's adds the residual u. The convolution runs in conv.cu, the layer in the
// library's route / projection / scan kernels.
#include <cstdio>

#include "conv.cuh"

namespace swimba {
cudaError_t run_block_gemm(bool bf16, int M, int N, int K, const void* A, int lda, const void* B, int ldb, void* C0,
                           int ldc0, void* C1, int ldc1, int split, const void* R, int ldr, void* status,
                           cudaStream_t s);
swimba_status api_check_dims(const swimba_dims* d);
swimba_status api_cuda_status(cudaError_t e);
void api_set_error(const char* msg);
}  // namespace swimba

using namespace swimba;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t up256(size_t v) { return (v + 255) & ~size_t(255); }
size_t io_bytes(int dtype) { return dtype == SWIMBA_BF16 ? 2 : 4; }

swimba_status check_conv(const swimba_dims* d, int32_t d_conv) {
  const swimba_status st = api_check_dims(d);
  if (st != SWIMBA_OK) return st;
  if (d_conv < 1 || d_conv > kMaxConvWidth) return SWIMBA_ERR_UNSUPPORTED;
  return SWIMBA_OK;
}

swimba_status check_block(const swimba_block_dims* bd) {
  if (bd == nullptr) return SWIMBA_ERR_INVALID_ARG;
  swimba_status st = check_conv(&bd->layer, bd->d_conv);
  if (st != SWIMBA_OK) return st;
  if (bd->d_model <= 0) return SWIMBA_ERR_INVALID_ARG;
  if (bd->d_model % 8 != 0 || bd->layer.io_dtype != bd->layer.w_dtype) return SWIMBA_ERR_UNSUPPORTED;
  if (bd->layer.batch * bd->layer.seqlen > INT32_MAX) return SWIMBA_ERR_UNSUPPORTED;
  return SWIMBA_OK;
}

// Workspace of the block: the layer's workspace first (its status block at offset 0), then the
// block's activations, each 256-byte aligned.
struct BlockLayout {
  size_t x_pre, z, x, y, idx, gates, delta, Bm, Cm, total;
};

BlockLayout block_layout(const swimba_block_dims* bd) {
  const swimba_dims& d = bd->layer;
  const size_t T = (size_t)(d.batch * d.seqlen), D = (size_t)d.d_inner, io = io_bytes(d.io_dtype);
  BlockLayout l{};
  size_t off = up256(swimba_workspace_size(&d, SWIMBA_OP_LAYER));
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = up256(off + bytes);
    return at;
  };
  l.x_pre = take(T * D * io);
  l.z = take(T * D * io);
  l.x = take(T * D * io);
  l.y = take(T * D * io);
  l.idx = take(T * d.top_k * 4);
  l.gates = take(T * d.top_k * 4);
  l.delta = take(T * D * 4);
  l.Bm = take(T * d.d_state * 4);
  l.Cm = take(T * d.d_state * 4);
  l.total = off;
  return l;
}

// Every argument a block call hands to the calls it makes, checked before the first launch (the
// layer's own calls check them again, but by then the in-projection would be queued).
swimba_status check_weights(const swimba_block_weights* w) {
  if (!w || !w->W_in || !w->conv_w || !w->conv_b || !w->W_out) return SWIMBA_ERR_INVALID_ARG;
  const swimba_weights& l = w->layer;
  if (!l.W_r || !l.W_x || !l.W_dt || !l.b_dt || !l.A || !l.D_skip) return SWIMBA_ERR_INVALID_ARG;
  if (!aligned16(w->W_in) || !aligned16(w->W_out) || !aligned16(w->conv_w) || !aligned16(w->conv_b))
    return SWIMBA_ERR_ALIGN;
  if (!aligned16(l.W_r) || !aligned16(l.W_x) || !aligned16(l.W_dt) || !aligned16(l.b_dt) || !aligned16(l.A) ||
      !aligned16(l.D_skip))
    return SWIMBA_ERR_ALIGN;
  return SWIMBA_OK;
}

swimba_status check_states(const swimba_block_dims* bd, const float* h0, const float* h_final, const void* cs_in,
                           const void* cs_out) {
  if (bd->d_conv > 1 && cs_in != nullptr && cs_in == cs_out) return SWIMBA_ERR_INVALID_ARG;
  if ((h0 && !aligned16(h0)) || (h_final && !aligned16(h_final))) return SWIMBA_ERR_ALIGN;
  if (bd->d_conv > 1 && ((cs_in && !aligned16(cs_in)) || (cs_out && !aligned16(cs_out)))) return SWIMBA_ERR_ALIGN;
  return SWIMBA_OK;
}

// in-projection: [x_pre | z] = u W_in, one GEMM whose epilogue writes columns [0, D) to x_pre and
// [D, 2D) to z
swimba_status in_proj(const swimba_block_dims* bd, const void* u, const swimba_block_weights* w, void* x_pre, void* z,
                      void* status, cudaStream_t s) {
  const swimba_dims& d = bd->layer;
  const bool bf16 = d.io_dtype == SWIMBA_BF16;
  const int M = (int)(d.batch * d.seqlen), D = d.d_inner, dm = bd->d_model;
  return api_cuda_status(
      run_block_gemm(bf16, M, 2 * D, dm, u, dm, w->W_in, 2 * D, x_pre, D, z, D, D, nullptr, 0, status, s));
}

// out-projection with the residual added in the GEMM's epilogue: out = y W_out + u (out may be u:
// every element is read and written by the same thread)
swimba_status out_proj(const swimba_block_dims* bd, const void* u, const swimba_block_weights* w, const void* y,
                       void* out, void* status, cudaStream_t s) {
  const swimba_dims& d = bd->layer;
  const int M = (int)(d.batch * d.seqlen), D = d.d_inner, dm = bd->d_model;
  return api_cuda_status(run_block_gemm(d.io_dtype == SWIMBA_BF16, M, dm, D, y, D, w->W_out, dm, out, dm, out, dm,
                                        dm, u, dm, status, s));
}

}  // namespace

extern "C" {

swimba_status swimba_conv1d_fwd(const swimba_dims* dims, int32_t d_conv, const void* x_pre, const float* conv_w,
                                const float* conv_b, const void* conv_state_in, void* x, void* conv_state_out,
                                void* stream) {
  const swimba_status st = check_conv(dims, d_conv);
  if (st != SWIMBA_OK) return st;
  if (!x_pre || !conv_w || !conv_b || !x) return SWIMBA_ERR_INVALID_ARG;
  if (d_conv > 1 && conv_state_in != nullptr && conv_state_in == conv_state_out) return SWIMBA_ERR_INVALID_ARG;
  if (!aligned16(x_pre) || !aligned16(x) || (d_conv > 1 && conv_state_in && !aligned16(conv_state_in)) ||
      (d_conv > 1 && conv_state_out && !aligned16(conv_state_out)))
    return SWIMBA_ERR_ALIGN;
  ConvParams p{dims->batch, dims->seqlen, dims->d_inner, d_conv, x_pre, conv_w, conv_b,
               d_conv > 1 ? conv_state_in : nullptr, x, d_conv > 1 ? conv_state_out : nullptr};
  return api_cuda_status(run_conv1d(p, dims->io_dtype == SWIMBA_BF16, false, static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_conv1d_step(const swimba_dims* dims, int32_t d_conv, const void* x_pre, const float* conv_w,
                                 const float* conv_b, void* conv_state, void* x, void* stream) {
  const swimba_status st = check_conv(dims, d_conv);
  if (st != SWIMBA_OK) return st;
  if (dims->seqlen != 1 || !x_pre || !conv_w || !conv_b || !x || (d_conv > 1 && !conv_state))
    return SWIMBA_ERR_INVALID_ARG;
  if (!aligned16(x_pre) || !aligned16(x) || (d_conv > 1 && !aligned16(conv_state))) return SWIMBA_ERR_ALIGN;
  ConvParams p{dims->batch, 1, dims->d_inner, d_conv, x_pre, conv_w, conv_b, nullptr, x,
               d_conv > 1 ? conv_state : nullptr};
  return api_cuda_status(run_conv1d(p, dims->io_dtype == SWIMBA_BF16, true, static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_block_gemm(int32_t dtype, int32_t M, int32_t N, int32_t K, const void* A, int32_t lda,
                                const void* B, int32_t ldb, void* C0, int32_t ldc0, void* C1, int32_t ldc1,
                                int32_t split, const void* R, int32_t ldr, void* ws, size_t ws_bytes,
                                void* stream) {
  if (dtype != SWIMBA_BF16 && dtype != SWIMBA_F32) return SWIMBA_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 1 || split < 0 || split > N) return SWIMBA_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < 256) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SWIMBA_ERR_ALIGN;
  if (M == 0 || N == 0) return SWIMBA_OK;
  if (!A || !B || lda < K || ldb < N || (split > 0 && (!C0 || ldc0 < split)) ||
      (split < N && (!C1 || ldc1 < N - split)) || (R && ldr < N))
    return SWIMBA_ERR_INVALID_ARG;
  const bool bf16 = dtype == SWIMBA_BF16;
  if (bf16) {
    if (N % 8 || split % 8 || lda % 8 || ldb % 8 || (split > 0 && ldc0 % 8) ||
        (split < N && ldc1 % 8) || (R && ldr % 8))
      return SWIMBA_ERR_UNSUPPORTED;
    if (!aligned16(A) || !aligned16(B) || (C0 && !aligned16(C0)) || (C1 && !aligned16(C1)) ||
        (R && !aligned16(R)))
      return SWIMBA_ERR_ALIGN;
  }
  return api_cuda_status(run_block_gemm(bf16, M, N, K, A, lda, B, ldb, C0, ldc0, C1, ldc1, split, R, ldr, ws,
                                        static_cast<cudaStream_t>(stream)));
}

size_t swimba_block_workspace_size(const swimba_block_dims* bd) {
  if (check_block(bd) != SWIMBA_OK) return 0;
  return block_layout(bd).total;
}

swimba_status swimba_block_fwd(const swimba_block_dims* bd, const void* u, const swimba_block_weights* w,
                               const float* h0, const void* conv_state_in, void* out, float* h_final,
                               void* conv_state_out, void* ws, size_t ws_bytes, void* stream) {
  swimba_status st = check_block(bd);
  if (st != SWIMBA_OK) return st;
  if (!u || !out) return SWIMBA_ERR_INVALID_ARG;
  if ((st = check_weights(w)) != SWIMBA_OK) return st;
  if ((st = check_states(bd, h0, h_final, conv_state_in, conv_state_out)) != SWIMBA_OK) return st;
  if (!aligned16(u) || !aligned16(out)) return SWIMBA_ERR_ALIGN;
  const BlockLayout l = block_layout(bd);
  if (ws == nullptr || ws_bytes < l.total) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SWIMBA_ERR_ALIGN;
  const swimba_dims* d = &bd->layer;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  void *x_pre = base + l.x_pre, *z = base + l.z, *x = base + l.x, *y = base + l.y;
  int32_t* idx = reinterpret_cast<int32_t*>(base + l.idx);
  float* gates = reinterpret_cast<float*>(base + l.gates);
  float* delta = reinterpret_cast<float*>(base + l.delta);
  float* Bm = reinterpret_cast<float*>(base + l.Bm);
  float* Cm = reinterpret_cast<float*>(base + l.Cm);
  const size_t layer_ws = swimba_workspace_size(d, SWIMBA_OP_LAYER);

  if ((st = in_proj(bd, u, w, x_pre, z, ws, s)) != SWIMBA_OK) return st;
  if ((st = swimba_conv1d_fwd(d, bd->d_conv, x_pre, w->conv_w, w->conv_b, conv_state_in, x, conv_state_out,
                              stream)) != SWIMBA_OK)
    return st;
  if ((st = swimba_route(d, x, w->layer.W_r, idx, gates, stream)) != SWIMBA_OK) return st;
  if ((st = swimba_mixed_proj(d, x, idx, gates, &w->layer, delta, Bm, Cm, ws, layer_ws, stream)) != SWIMBA_OK)
    return st;
  if ((st = swimba_scan_fwd(d, x, z, delta, Bm, Cm, idx, gates, &w->layer, h0, y, h_final, nullptr, ws, layer_ws,
                            stream)) != SWIMBA_OK)
    return st;
  return out_proj(bd, u, w, y, out, ws, s);
}

swimba_status swimba_block_step(const swimba_block_dims* bd, const void* u, const swimba_block_weights* w, float* h,
                                void* conv_state, void* out, void* ws, size_t ws_bytes, void* stream) {
  swimba_status st = check_block(bd);
  if (st != SWIMBA_OK) return st;
  if (bd->layer.seqlen != 1 || !u || !out || !h || (bd->d_conv > 1 && !conv_state)) return SWIMBA_ERR_INVALID_ARG;
  if ((st = check_weights(w)) != SWIMBA_OK) return st;
  if ((st = check_states(bd, h, nullptr, conv_state, nullptr)) != SWIMBA_OK) return st;
  if (!aligned16(u) || !aligned16(out)) return SWIMBA_ERR_ALIGN;
  const BlockLayout l = block_layout(bd);
  if (ws == nullptr || ws_bytes < l.total) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SWIMBA_ERR_ALIGN;
  const swimba_dims* d = &bd->layer;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  void *x_pre = base + l.x_pre, *z = base + l.z, *x = base + l.x, *y = base + l.y;
  int32_t* idx = reinterpret_cast<int32_t*>(base + l.idx);
  float* gates = reinterpret_cast<float*>(base + l.gates);
  float* delta = reinterpret_cast<float*>(base + l.delta);
  float* Bm = reinterpret_cast<float*>(base + l.Bm);
  float* Cm = reinterpret_cast<float*>(base + l.Cm);
  const size_t layer_ws = swimba_workspace_size(d, SWIMBA_OP_LAYER);

  if ((st = in_proj(bd, u, w, x_pre, z, ws, s)) != SWIMBA_OK) return st;
  if ((st = swimba_conv1d_step(d, bd->d_conv, x_pre, w->conv_w, w->conv_b, conv_state, x, stream)) != SWIMBA_OK)
    return st;
  if ((st = swimba_route(d, x, w->layer.W_r, idx, gates, stream)) != SWIMBA_OK) return st;
  if ((st = swimba_mixed_proj(d, x, idx, gates, &w->layer, delta, Bm, Cm, ws, layer_ws, stream)) != SWIMBA_OK)
    return st;
  if ((st = swimba_step(d, x, z, delta, Bm, Cm, idx, gates, &w->layer, h, y, stream)) != SWIMBA_OK) return st;
  return out_proj(bd, u, w, y, out, ws, s);
}

}  // extern "C"
