// C-ABI plumbing of libnf4ls: status messages, the shard format and its quantiser
// entry point, header checks and process-wide options.
//
// Shard format: "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" §2.1 (per-layer offline
// shards of packed bytes plus absmax, nested absmax and offset sidecars) and the
// cache key of the layer-streaming review ("4GB 显存微调 8B 模型是真的", mechanism
// section: keyed by quantisation method and source checkpoint fingerprint, so the
// wrong bytes are never streamed).  §2.4: the code tables are asserted constant,
// which the header's code-table hash enforces.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <vector>

#include "internal.h"

namespace nf4ls {

namespace {
thread_local char g_msg[1024] = "";
int g_gemm_path = 0;
int g_gemm_pair = 1;
int g_gemm_half = 0;  // 0 auto, 1 never, 2 always, 3 the last partial wave only
int g_attn_tc = 1;    // attention forward on tcgen05 where the shape allows
}  // namespace

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return status;
}

void clear_error() { g_msg[0] = 0; }

int gemm_path() { return g_gemm_path; }
int gemm_pair() { return g_gemm_pair; }
int gemm_half_mode() { return g_gemm_half; }
int attention_tc() { return g_attn_tc; }

void shard_layout(const nf4ls_layer_cfg* c, ShardLayout* L) {
  const int qd = c->n_q * c->head_dim, kvd = c->n_kv * c->head_dim;
  const int rows[7] = {qd, kvd, kvd, c->hidden, c->inter, c->inter, c->hidden};
  const int cols[7] = {c->hidden, c->hidden, c->hidden, qd, c->hidden, c->hidden, c->inter};
  uint64_t off = 1024;  // header [0,256) + descriptors [256,832), data from 1024
  uint64_t q = 0;
  for (int t = 0; t < 7; ++t) {
    const uint64_t n = (uint64_t)rows[t] * cols[t];
    const uint64_t nb = n / 64, ng = (nb + 255) / 256;
    L->rows[t] = rows[t];
    L->cols[t] = cols[t];
    L->off_packed[t] = off;
    off = round_up(off + n / 2, 256);
    L->off_q8[t] = off;
    off = round_up(off + nb, 256);
    L->off_nested[t] = off;
    off = round_up(off + 4 * ng, 256);
    L->off_offset[t] = off;
    off = round_up(off + 4, 256);
    q += n / 2 + nb + 4 * ng + 4;
  }
  L->off_norm_in = off;
  off = round_up(off + 2ull * c->hidden, 256);
  L->off_norm_post = off;
  off = round_up(off + 2ull * c->hidden, 256);
  L->total = off;
  L->quantized = q;
}

void shard_view(const nf4ls_layer_cfg* cfg, const void* shard_dev, ShardView* v) {
  ShardLayout L;
  shard_layout(cfg, &L);
  const uint8_t* b = static_cast<const uint8_t*>(shard_dev);
  for (int t = 0; t < 7; ++t) {
    v->t[t].packed = b + L.off_packed[t];
    v->t[t].q8 = b + L.off_q8[t];
    v->t[t].nested = reinterpret_cast<const float*>(b + L.off_nested[t]);
    v->t[t].offset = reinterpret_cast<const float*>(b + L.off_offset[t]);
    v->t[t].rows = L.rows[t];
    v->t[t].cols = L.cols[t];
  }
  v->norm_in = reinterpret_cast<const __nv_bfloat16*>(b + L.off_norm_in);
  v->norm_post = reinterpret_cast<const __nv_bfloat16*>(b + L.off_norm_post);
}

int check_cfg(const nf4ls_layer_cfg* c) {
  if (!c) return fail(NF4LS_INVALID_ARG, "null layer config");
  if (c->hidden <= 0 || c->inter <= 0 || c->n_q <= 0 || c->n_kv <= 0 || c->head_dim <= 0 || c->batch <= 0 ||
      c->seq <= 0)
    return fail(NF4LS_SHAPE, "layer config has a non-positive dimension");
  if (c->head_dim != 64 && c->head_dim != 128) return fail(NF4LS_SHAPE, "head_dim must be 64 or 128");
  if (c->n_q % c->n_kv) return fail(NF4LS_SHAPE, "n_q must be a multiple of n_kv");
  if (c->hidden % 64 || c->inter % 128) return fail(NF4LS_SHAPE, "hidden % 64 and inter % 128 must be 0");
  if ((c->n_kv * c->head_dim) % 64) return fail(NF4LS_SHAPE, "kv width must be a multiple of 64");
  if (c->lora_r != 16) return fail(NF4LS_SHAPE, "lora_r must be 16");
  return NF4LS_OK;
}

}  // namespace nf4ls

using namespace nf4ls;

extern "C" const char* nf4ls_last_error(void) { return g_msg; }
extern "C" int nf4ls_version(void) { return 1; }

extern "C" int nf4ls_set_gemm_path(int path) {
  if (path != 0 && path != 1) return fail(NF4LS_INVALID_ARG, "gemm path must be 0 or 1");
  g_gemm_path = path;
  return NF4LS_OK;
}

extern "C" int nf4ls_set_gemm_pair(int on) {
  g_gemm_pair = on ? 1 : 0;
  return NF4LS_OK;
}

extern "C" int nf4ls_set_attention_path(int tc) {
  g_attn_tc = tc ? 1 : 0;
  return NF4LS_OK;
}

extern "C" int nf4ls_set_gemm_half(int mode) {
  clear_error();
  if (mode < 0 || mode > 3) return fail(NF4LS_INVALID_ARG, "nf4ls_set_gemm_half: mode %d not in 0..3", mode);
  g_gemm_half = mode;
  return NF4LS_OK;
}

extern "C" size_t nf4ls_shard_bytes(const nf4ls_layer_cfg* cfg) {
  if (!cfg) return 0;
  ShardLayout L;
  shard_layout(cfg, &L);
  return L.total;
}

extern "C" size_t nf4ls_shard_quantized_bytes(const nf4ls_layer_cfg* cfg) {
  if (!cfg) return 0;
  ShardLayout L;
  shard_layout(cfg, &L);
  return L.quantized;
}

extern "C" size_t nf4ls_shard_scratch_bytes(const nf4ls_layer_cfg* cfg) {
  if (!cfg) return 0;
  ShardLayout L;
  shard_layout(cfg, &L);
  size_t mx = 0;
  for (int t = 0; t < 7; ++t) {
    const size_t n = (size_t)L.rows[t] * L.cols[t];
    mx = n > mx ? n : mx;
  }
  return nf4ls_quantize_scratch_bytes(mx);
}

extern "C" int nf4_quantize_shard(const nf4ls_layer_cfg* cfg, const void* const* w, uint64_t fingerprint,
                                  void* shard_dev, size_t cap, size_t* used, void* scratch_dev, size_t scratch_bytes,
                                  nf4ls_stream stream) {
  clear_error();
  NF4_TRY(check_cfg(cfg));
  if (!w || !shard_dev || !scratch_dev) return fail(NF4LS_INVALID_ARG, "nf4_quantize_shard: null pointer");
  for (int t = 0; t < NF4LS_N_TENSORS; ++t)
    if (!w[t]) return fail(NF4LS_INVALID_ARG, "nf4_quantize_shard: weight %d is null", t);
  if (!aligned(shard_dev, 256)) return fail(NF4LS_ALIGN, "nf4_quantize_shard: shard must be 256-byte aligned");
  ShardLayout L;
  shard_layout(cfg, &L);
  if (cap < L.total) return fail(NF4LS_INVALID_ARG, "nf4_quantize_shard: cap %zu < %llu", cap,
                                 (unsigned long long)L.total);
  if (scratch_bytes < nf4ls_shard_scratch_bytes(cfg))
    return fail(NF4LS_INVALID_ARG, "nf4_quantize_shard: scratch too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(shard_dev);

  // Header and descriptors are staged on the host and copied with the stream.
  std::vector<uint8_t> hdr(1024, 0);
  nf4ls_shard_header* h = reinterpret_cast<nf4ls_shard_header*>(hdr.data());
  h->magic = NF4LS_SHARD_MAGIC;
  h->version = NF4LS_SHARD_VERSION;
  h->method = NF4LS_METHOD_NF4_DQ;
  h->blocksize = 64;
  h->nested_blocksize = 256;
  h->n_tensors = NF4LS_N_TENSORS;
  h->hidden = cfg->hidden;
  h->inter = cfg->inter;
  h->n_q = cfg->n_q;
  h->n_kv = cfg->n_kv;
  h->head_dim = cfg->head_dim;
  h->codebook_hash = codebooks().hash;
  h->fingerprint = fingerprint;
  h->total_bytes = L.total;
  h->quantized_bytes = L.quantized;
  nf4ls_tensor_desc* d = reinterpret_cast<nf4ls_tensor_desc*>(hdr.data() + 256);
  for (int t = 0; t < 7; ++t) {
    d[t].kind = t;
    d[t].format = 1;
    d[t].rows = L.rows[t];
    d[t].cols = L.cols[t];
    d[t].off_packed = L.off_packed[t];
    d[t].off_q8 = L.off_q8[t];
    d[t].off_nested = L.off_nested[t];
    d[t].off_offset = L.off_offset[t];
  }
  for (int t = 7; t < 9; ++t) {
    d[t].kind = t;
    d[t].format = 2;
    d[t].rows = 1;
    d[t].cols = cfg->hidden;
    d[t].off_packed = t == 7 ? L.off_norm_in : L.off_norm_post;
  }
  // Zero the whole shard first so padding bytes are deterministic.
  NF4_CUDA_TRY(cudaMemsetAsync(base, 0, L.total, s));
  NF4_CUDA_TRY(cudaMemcpyAsync(base, hdr.data(), hdr.size(), cudaMemcpyHostToDevice, s));
  for (int t = 0; t < 7; ++t) {
    const size_t n = (size_t)L.rows[t] * L.cols[t];
    NF4_TRY(quantize_tensor(w[t], n, base + L.off_packed[t], base + L.off_q8[t],
                            reinterpret_cast<float*>(base + L.off_nested[t]),
                            reinterpret_cast<float*>(base + L.off_offset[t]), scratch_dev, scratch_bytes, s));
  }
  NF4_CUDA_TRY(cudaMemcpyAsync(base + L.off_norm_in, w[7], 2ull * cfg->hidden, cudaMemcpyDeviceToDevice, s));
  NF4_CUDA_TRY(cudaMemcpyAsync(base + L.off_norm_post, w[8], 2ull * cfg->hidden, cudaMemcpyDeviceToDevice, s));
  // The header is a pageable host buffer: make sure the copy has consumed it.
  NF4_CUDA_TRY(cudaStreamSynchronize(s));
  if (used) *used = L.total;
  return NF4LS_OK;
}

extern "C" int nf4ls_shard_check(const void* header_host, const nf4ls_layer_cfg* cfg, uint64_t expected_fp) {
  clear_error();
  if (!header_host) return fail(NF4LS_INVALID_ARG, "null header");
  const nf4ls_shard_header* h = static_cast<const nf4ls_shard_header*>(header_host);
  if (h->magic != NF4LS_SHARD_MAGIC || h->version != NF4LS_SHARD_VERSION)
    return fail(NF4LS_INVALID_ARG, "not an NF4 shard (magic %08x version %u)", h->magic, h->version);
  if (h->method != NF4LS_METHOD_NF4_DQ || h->blocksize != 64 || h->nested_blocksize != 256)
    return fail(NF4LS_INVALID_ARG, "unsupported quantisation method %u", h->method);
  if (h->codebook_hash != codebooks().hash)
    return fail(NF4LS_CODEBOOK_MISMATCH, "shard code tables %016llx differ from the library's %016llx",
                (unsigned long long)h->codebook_hash, (unsigned long long)codebooks().hash);
  if (expected_fp && h->fingerprint != expected_fp)
    return fail(NF4LS_FINGERPRINT_MISMATCH, "shard fingerprint %016llx, expected %016llx",
                (unsigned long long)h->fingerprint, (unsigned long long)expected_fp);
  if (cfg) {
    if ((int)h->hidden != cfg->hidden || (int)h->inter != cfg->inter || (int)h->n_q != cfg->n_q ||
        (int)h->n_kv != cfg->n_kv || (int)h->head_dim != cfg->head_dim)
      return fail(NF4LS_SHAPE, "shard dimensions differ from the layer config");
    if (h->total_bytes != nf4ls_shard_bytes(cfg)) return fail(NF4LS_SHAPE, "shard size differs");
  }
  return NF4LS_OK;
}
