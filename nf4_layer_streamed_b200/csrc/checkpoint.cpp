// Adapter checkpoint / resume.  The trainable state of the run is the LoRA adapter
// (A and B of every adapted projection, fp32), the AdamW moments and the step count
// that drives the bias correction; the NF4 base is frozen and comes back from its
// own shards.  "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" §3.2 records a release whose
// adapters were written correctly during training but read back as empty, and no
// test had saved an adapter and loaded it again: here the loader refuses any file
// whose shapes, size or checksum do not match, before it touches the device, and
// a resumed run continues bit for bit.
//
// File layout (little-endian): a 64-byte AdapterHeader, then three arrays of
// n_floats fp32 each, in the order LoRA parameters, AdamW first moment, AdamW
// second moment.  Each array is the device layout as is: n_layers blocks of
// nf4ls_lora_stride floats, [A_q | B_q | A_v | B_v] per layer.  The header's
// checksum is 64-bit FNV-1a over the header itself (with the checksum field set to
// zero) and then the three arrays' bytes in file order, so a damaged step count or
// alpha is refused like a damaged array.
#include <errno.h>
#include <fcntl.h>
#include <stdio.h>
#include <string.h>
#include <unistd.h>

#include <string>
#include <vector>

#include "internal.h"

namespace nf4ls {
namespace {

struct AdapterHeader {
  uint32_t magic;
  uint32_t version;
  int32_t hidden, inter, n_q, n_kv, head_dim, lora_r, n_layers;
  float lora_alpha;
  int32_t step;
  uint32_t reserved;
  uint64_t n_floats;  // per array
  uint64_t checksum;
};
static_assert(sizeof(AdapterHeader) == 64, "adapter header is 64 bytes");

uint64_t fnv1a64(const void* data, size_t n, uint64_t h) {
  const auto* b = static_cast<const uint8_t*>(data);
  for (size_t i = 0; i < n; ++i) {
    h ^= b[i];
    h *= 0x100000001B3ull;
  }
  return h;
}
constexpr uint64_t kFnvBasis = 0xCBF29CE484222325ull;

uint64_t file_checksum(const AdapterHeader& h, const float* arrays, size_t n_bytes) {
  AdapterHeader z = h;
  z.checksum = 0;
  return fnv1a64(arrays, n_bytes, fnv1a64(&z, sizeof z, kFnvBasis));
}

// Makes a completed rename durable: the new directory entry is on disk once the
// directory itself has been flushed.
int fsync_parent_dir(const char* path) {
  std::string dir(path);
  const size_t slash = dir.find_last_of('/');
  dir = slash == std::string::npos ? std::string(".") : (slash == 0 ? std::string("/") : dir.substr(0, slash));
  const int fd = ::open(dir.c_str(), O_RDONLY | O_DIRECTORY | O_CLOEXEC);
  if (fd < 0) return -1;
  const int r = ::fsync(fd);
  ::close(fd);
  return r;
}

int check_args(const char* path, const nf4ls_model_cfg* c, const nf4ls_model* m, const char* who) {
  if (!path || !*path || !c || !m) return fail(NF4LS_INVALID_ARG, "%s: null path, config or model", who);
  if (!m->lora_dev || !m->adam_m_dev || !m->adam_v_dev)
    return fail(NF4LS_INVALID_ARG, "%s: model needs lora_dev, adam_m_dev and adam_v_dev", who);
  if (c->n_layers <= 0 || nf4ls_lora_stride(&c->layer) == 0)
    return fail(NF4LS_SHAPE, "%s: empty adapter (n_layers %d, lora_r %d)", who, c->n_layers, c->layer.lora_r);
  return NF4LS_OK;
}

size_t floats_of(const nf4ls_model_cfg* c) { return (size_t)c->n_layers * nf4ls_lora_stride(&c->layer); }

int write_all(int fd, const void* p, size_t n) {
  const auto* b = static_cast<const uint8_t*>(p);
  while (n) {
    const ssize_t w = ::write(fd, b, n);
    if (w < 0 && errno == EINTR) continue;
    if (w <= 0) return -1;
    b += w;
    n -= (size_t)w;
  }
  return 0;
}

int read_all(int fd, void* p, size_t n) {
  auto* b = static_cast<uint8_t*>(p);
  while (n) {
    const ssize_t r = ::read(fd, b, n);
    if (r < 0 && errno == EINTR) continue;
    if (r <= 0) return -1;
    b += r;
    n -= (size_t)r;
  }
  return 0;
}

}  // namespace
}  // namespace nf4ls

using namespace nf4ls;

extern "C" size_t nf4ls_adapter_file_bytes(const nf4ls_model_cfg* cfg) {
  if (!cfg || cfg->n_layers <= 0) return 0;
  return sizeof(AdapterHeader) + 3 * floats_of(cfg) * sizeof(float);
}

extern "C" int nf4ls_adapter_save(const char* path, const nf4ls_model_cfg* cfg, const nf4ls_model* model,
                                  int32_t step, nf4ls_stream stream) {
  clear_error();
  NF4_TRY(check_args(path, cfg, model, "nf4ls_adapter_save"));
  if (step < 0) return fail(NF4LS_INVALID_ARG, "nf4ls_adapter_save: step %d < 0", step);
  const size_t n = floats_of(cfg);
  std::vector<float> host(3 * n);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Ordered after every step queued on the stream, so the state saved is the one
  // the last queued AdamW update wrote.
  const float* src[3] = {model->lora_dev, model->adam_m_dev, model->adam_v_dev};
  for (int a = 0; a < 3; ++a)
    NF4_CUDA_TRY(cudaMemcpyAsync(host.data() + a * n, src[a], n * sizeof(float), cudaMemcpyDeviceToHost, s));
  NF4_CUDA_TRY(cudaStreamSynchronize(s));

  AdapterHeader h{};
  h.magic = NF4LS_ADAPTER_MAGIC;
  h.version = NF4LS_ADAPTER_VERSION;
  h.hidden = cfg->layer.hidden;
  h.inter = cfg->layer.inter;
  h.n_q = cfg->layer.n_q;
  h.n_kv = cfg->layer.n_kv;
  h.head_dim = cfg->layer.head_dim;
  h.lora_r = cfg->layer.lora_r;
  h.n_layers = cfg->n_layers;
  h.lora_alpha = cfg->layer.lora_alpha;
  h.step = step;
  h.n_floats = n;
  h.checksum = file_checksum(h, host.data(), host.size() * sizeof(float));

  // Written under a temporary name and renamed into place, so a crash mid-write
  // leaves the previous checkpoint intact.
  const std::string tmp = std::string(path) + ".tmp";
  const int fd = ::open(tmp.c_str(), O_WRONLY | O_CREAT | O_TRUNC | O_CLOEXEC, 0644);
  if (fd < 0) return fail(NF4LS_IO, "nf4ls_adapter_save: open %s: %s", tmp.c_str(), strerror(errno));
  const bool ok = write_all(fd, &h, sizeof h) == 0 && write_all(fd, host.data(), host.size() * sizeof(float)) == 0 &&
                  ::fsync(fd) == 0;
  const int err = errno;
  ::close(fd);
  if (!ok) {
    ::unlink(tmp.c_str());
    return fail(NF4LS_IO, "nf4ls_adapter_save: write %s: %s", tmp.c_str(), strerror(err));
  }
  if (::rename(tmp.c_str(), path) != 0) {
    const int e = errno;
    ::unlink(tmp.c_str());
    return fail(NF4LS_IO, "nf4ls_adapter_save: rename to %s: %s", path, strerror(e));
  }
  if (fsync_parent_dir(path) != 0)
    return fail(NF4LS_IO, "nf4ls_adapter_save: flushing the directory of %s: %s", path, strerror(errno));
  return NF4LS_OK;
}

extern "C" int nf4ls_adapter_load(const char* path, const nf4ls_model_cfg* cfg, const nf4ls_model* model,
                                  int32_t* step, nf4ls_stream stream) {
  clear_error();
  NF4_TRY(check_args(path, cfg, model, "nf4ls_adapter_load"));
  if (!step) return fail(NF4LS_INVALID_ARG, "nf4ls_adapter_load: null step");
  const int fd = ::open(path, O_RDONLY | O_CLOEXEC);
  if (fd < 0) return fail(NF4LS_IO, "nf4ls_adapter_load: open %s: %s", path, strerror(errno));
  AdapterHeader h{};
  if (read_all(fd, &h, sizeof h) != 0) {
    ::close(fd);
    return fail(NF4LS_IO, "nf4ls_adapter_load: %s is shorter than the header", path);
  }
  if (h.magic != NF4LS_ADAPTER_MAGIC || h.version != NF4LS_ADAPTER_VERSION) {
    ::close(fd);
    return fail(NF4LS_INVALID_ARG, "nf4ls_adapter_load: %s is not an adapter checkpoint (magic %08x version %u)", path,
                h.magic, h.version);
  }
  const nf4ls_layer_cfg& l = cfg->layer;
  if (h.hidden != l.hidden || h.inter != l.inter || h.n_q != l.n_q || h.n_kv != l.n_kv || h.head_dim != l.head_dim ||
      h.lora_r != l.lora_r || h.n_layers != cfg->n_layers || h.lora_alpha != l.lora_alpha) {
    ::close(fd);
    return fail(NF4LS_SHAPE,
                "nf4ls_adapter_load: %s holds H %d I %d heads %d/%d d %d r %d alpha %g, %d layers; the model has "
                "H %d I %d heads %d/%d d %d r %d alpha %g, %d layers",
                path, h.hidden, h.inter, h.n_q, h.n_kv, h.head_dim, h.lora_r, (double)h.lora_alpha, h.n_layers,
                l.hidden, l.inter, l.n_q, l.n_kv, l.head_dim, l.lora_r, (double)l.lora_alpha, cfg->n_layers);
  }
  const size_t n = floats_of(cfg);
  if (h.n_floats != n || h.step < 0) {
    ::close(fd);
    return fail(NF4LS_SHAPE, "nf4ls_adapter_load: %s: %llu floats per array, step %d (expected %zu floats)", path,
                (unsigned long long)h.n_floats, h.step, n);
  }
  std::vector<float> host(3 * n);
  const int rd = read_all(fd, host.data(), host.size() * sizeof(float));
  uint8_t extra;
  const bool trailing = rd == 0 && ::read(fd, &extra, 1) > 0;
  ::close(fd);
  if (rd != 0) return fail(NF4LS_IO, "nf4ls_adapter_load: %s is truncated", path);
  if (trailing) return fail(NF4LS_IO, "nf4ls_adapter_load: %s has bytes after the last array", path);
  if (file_checksum(h, host.data(), host.size() * sizeof(float)) != h.checksum)
    return fail(NF4LS_IO, "nf4ls_adapter_load: %s fails its checksum", path);

  // Every check has passed: only now is the device state overwritten.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* dst[3] = {model->lora_dev, model->adam_m_dev, model->adam_v_dev};
  for (int a = 0; a < 3; ++a)
    NF4_CUDA_TRY(cudaMemcpyAsync(dst[a], host.data() + a * n, n * sizeof(float), cudaMemcpyHostToDevice, s));
  NF4_CUDA_TRY(cudaStreamSynchronize(s));  // the host buffer dies on return
  *step = h.step;
  return NF4LS_OK;
}
