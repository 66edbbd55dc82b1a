// Streaming pool: n-deep HBM slot pool fed from the pinned host store on a
// dedicated copy stream.
//
// Mechanism from the layer-streaming review ("4GB 显存微调 8B 模型是真的", mechanism
// section, and its English version): the frozen base lives in page-locked host
// memory, 2-8 preallocated device buffers (two by default) are filled
// asynchronously on their own CUDA stream, prefetching layer i+1 during the forward
// and layer i-1 during the backward, so that copies overlap compute.
//
// Reuse rule from the same page's bug history (Issue #331: a weight kept alive
// outside save_for_backward aliased a pooled buffer and silently corrupted the
// gradients of >165 MiB layers): a slot is overwritten only after the event that
// its releaser recorded on the compute stream -- after every kernel that reads the
// slot -- has completed.  The copy stream waits on that event; nothing else orders
// the reuse.  A layer still held by a slot is served without a new copy, which lets
// the backward start on the layers the forward left behind.
//
// Disk source (same pages, mechanism section: the base falls back from pinned memory
// to an NVMe disk when memory is short; SATA and spinning disks are refused): the
// store is a file, a reader thread reads each requested layer into one of two
// caller-owned pinned staging buffers and enqueues its copy into the slot on the copy
// stream; the slot rules above are unchanged.
#include <dlfcn.h>
#include <fcntl.h>
#include <nccl.h>
#include <sys/stat.h>
#include <sys/sysmacros.h>
#include <unistd.h>

#include <algorithm>
#include <chrono>
#include <climits>
#include <condition_variable>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <deque>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include "internal.h"

using namespace nf4ls;

namespace {

constexpr size_t kIoAlign = 4096;
constexpr int kFillWaitMs = 60000;  // host bound on waiting for a layer's file read

size_t io_round(size_t b) { return (b + kIoAlign - 1) / kIoAlign * kIoAlign; }

// Reads [off, off + need) of fd into dst (need <= cap, cap a multiple of 4096 when
// direct); returns 0 or errno-like failure.
int read_range(int fd, bool direct, uint8_t* dst, size_t cap, size_t off, size_t need) {
  size_t done = 0;
  const size_t want = direct ? std::min(cap, io_round(need)) : need;
  while (done < need) {
    const ssize_t r = pread(fd, dst + done, want - done, (off_t)(off + done));
    if (r < 0) {
      if (errno == EINTR) continue;
      return errno ? errno : EIO;
    }
    if (r == 0) return EIO;  // the file ends before the layer does
    done += (size_t)r;
  }
  return 0;
}

}  // namespace

// NCCL, resolved at run time from the copy already in the process (the one torch
// loaded) or else from the system's libnccl.so.2.
struct NcclApi {
  ncclResult_t (*get_unique_id)(ncclUniqueId*) = nullptr;
  ncclResult_t (*comm_init_rank)(ncclComm_t*, int, ncclUniqueId, int) = nullptr;
  ncclResult_t (*broadcast)(const void*, void*, size_t, ncclDataType_t, int, ncclComm_t, cudaStream_t) = nullptr;
  ncclResult_t (*comm_destroy)(ncclComm_t) = nullptr;
  const char* (*error_string)(ncclResult_t) = nullptr;
  bool ok = false;
};

const NcclApi& nccl_api() {
  static NcclApi a = [] {
    NcclApi r;
    void* h = dlopen("libnccl.so.2", RTLD_NOW | RTLD_NOLOAD);
    if (!h) h = dlopen("libnccl.so.2", RTLD_NOW);
    if (!h) return r;
    r.get_unique_id = reinterpret_cast<decltype(r.get_unique_id)>(dlsym(h, "ncclGetUniqueId"));
    r.comm_init_rank = reinterpret_cast<decltype(r.comm_init_rank)>(dlsym(h, "ncclCommInitRank"));
    r.broadcast = reinterpret_cast<decltype(r.broadcast)>(dlsym(h, "ncclBroadcast"));
    r.comm_destroy = reinterpret_cast<decltype(r.comm_destroy)>(dlsym(h, "ncclCommDestroy"));
    r.error_string = reinterpret_cast<decltype(r.error_string)>(dlsym(h, "ncclGetErrorString"));
    r.ok = r.get_unique_id && r.comm_init_rank && r.broadcast && r.comm_destroy && r.error_string;
    return r;
  }();
  return a;
}

struct FileSource {
  int fd = -1;
  bool direct = false;
  uint8_t* staging[2] = {nullptr, nullptr};
  size_t staging_each = 0;
  cudaEvent_t staged[2] = {nullptr, nullptr};  // the copy out of staging buffer b is done
  bool staged_recorded[2] = {false, false};
  uint64_t seq = 0;
  struct Job {
    int layer, slot;
    bool wait_freed;
  };
  std::deque<Job> jobs;
  std::condition_variable cv_job, cv_done;
  bool stop = false;
  int error = NF4LS_OK;
  std::string error_msg;
  std::thread reader;
};

struct nf4ls_pool {
  int device = 0;
  const uint8_t* store = nullptr;
  std::vector<size_t> off, bytes;
  int n_layers = 0, depth = 0;
  uint8_t* slots = nullptr;
  size_t slot_bytes = 0;
  cudaStream_t copy = nullptr;
  // Which layer each slot holds, hits, reuse order and ownership: the host-only plan.
  // What the device sees of a slot: its events.
  SlotPlan plan;
  struct Slot {
    bool filling = false;  // disk source: the reader has not enqueued this slot's copy yet
    cudaEvent_t ready = nullptr, freed = nullptr;
  };
  std::vector<Slot> slot;
  bool poison = false;
  nf4ls_pool_stats stats{};
  std::mutex mu;
  FileSource* file = nullptr;
  // layer-sharded fetch: the owner of layer l is rank l % world
  ncclComm_t comm = nullptr;
  int rank = 0, world = 1;

  int find(int layer) const { return plan.find(layer); }

  int issue(int layer, int* out_idx) {
    PlanStep st;
    NF4_TRY(plan.preview(layer, &st));
    *out_idx = st.slot;
    if (!st.fill) return NF4LS_OK;
    if (file && file->error) return fail(file->error, "pool: disk source failed earlier: %s", file->error_msg.c_str());
    NF4_TRY(plan.issue(layer, &st));
    Slot& s = slot[st.slot];
    uint8_t* dst = slots + (size_t)st.slot * slot_bytes;
    if (file) {  // the reader thread reads the layer and enqueues the copy
      file->jobs.push_back(FileSource::Job{layer, st.slot, st.after_release});
      file->cv_job.notify_one();
      s.filling = true;
      stats.bytes_copied += bytes[layer];
      stats.copies += 1;
      return NF4LS_OK;
    }
    if (st.after_release) NF4_CUDA_TRY(cudaStreamWaitEvent(copy, s.freed, 0));
    if (poison) NF4_CUDA_TRY(cudaMemsetAsync(dst, 0xFF, slot_bytes, copy));
    if (st.host_read) {
      NF4_CUDA_TRY(cudaMemcpyAsync(dst, store + off[layer], bytes[layer], cudaMemcpyHostToDevice, copy));
      stats.bytes_copied += bytes[layer];
      stats.copies += 1;
    }
    if (st.broadcast) {  // from the owner's slot into every other rank's slot, in place
      const ncclResult_t r = nccl_api().broadcast(dst, dst, bytes[layer], ncclUint8, st.owner, comm, copy);
      if (r != ncclSuccess) return fail(NF4LS_CUDA, "pool: NCCL broadcast of layer %d: %s", layer,
                                        nccl_api().error_string(r));
      if (!st.host_read) stats.peer_bytes += bytes[layer];
    }
    NF4_CUDA_TRY(cudaEventRecord(s.ready, copy));
    return NF4LS_OK;
  }

  // Disk source: waits (lk held on mu) until slot idx's copy has been enqueued.
  int wait_filled(std::unique_lock<std::mutex>& lk, int idx) {
    if (!file) return NF4LS_OK;
    const bool ok = file->cv_done.wait_for(lk, std::chrono::milliseconds(kFillWaitMs),
                                           [&] { return !slot[idx].filling || file->error != NF4LS_OK; });
    if (file->error) return fail(file->error, "pool: disk source: %s", file->error_msg.c_str());
    if (!ok) return fail(NF4LS_TIMEOUT, "pool: layer %d not read from disk after %d ms", plan.layer_in(idx), kFillWaitMs);
    return NF4LS_OK;
  }

  void reader_loop() {
    cudaSetDevice(device);
    FileSource& f = *file;
    while (true) {
      FileSource::Job j;
      {
        std::unique_lock<std::mutex> lk(mu);
        f.cv_job.wait(lk, [&] { return f.stop || !f.jobs.empty(); });
        if (f.jobs.empty()) return;  // stop requested and nothing left
        j = f.jobs.front();
      }
      const int b = (int)(f.seq++ & 1);
      int err = NF4LS_OK;
      std::string msg;
      if (f.staged_recorded[b]) {  // the previous copy out of this staging buffer must be done
        const auto t0 = std::chrono::steady_clock::now();
        while (true) {
          const cudaError_t e = cudaEventQuery(f.staged[b]);
          if (e == cudaSuccess) break;
          if (e != cudaErrorNotReady) {
            err = NF4LS_CUDA;
            msg = cudaGetErrorString(e);
            break;
          }
          if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(kFillWaitMs)) {
            err = NF4LS_TIMEOUT;
            msg = "staging buffer copy did not finish";
            break;
          }
          std::this_thread::sleep_for(std::chrono::microseconds(20));
        }
      }
      if (!err) {
        const int r = read_range(f.fd, f.direct, f.staging[b], f.staging_each, off[j.layer], bytes[j.layer]);
        if (r) {
          err = NF4LS_IO;
          msg = std::string("read of layer ") + std::to_string(j.layer) + ": " + strerror(r);
        }
      }
      std::lock_guard<std::mutex> g(mu);
      f.jobs.pop_front();
      Slot& s = slot[j.slot];
      if (!err) {
        uint8_t* dst = slots + (size_t)j.slot * slot_bytes;
        cudaError_t e = cudaSuccess;
        if (j.wait_freed) e = cudaStreamWaitEvent(copy, s.freed, 0);
        if (e == cudaSuccess && poison) e = cudaMemsetAsync(dst, 0xFF, slot_bytes, copy);
        if (e == cudaSuccess) e = cudaMemcpyAsync(dst, f.staging[b], bytes[j.layer], cudaMemcpyHostToDevice, copy);
        if (e == cudaSuccess) e = cudaEventRecord(f.staged[b], copy);
        if (e == cudaSuccess) e = cudaEventRecord(s.ready, copy);
        if (e != cudaSuccess) {
          err = NF4LS_CUDA;
          msg = cudaGetErrorString(e);
        }
        f.staged_recorded[b] = true;
      }
      if (err && !f.error) {
        f.error = err;
        f.error_msg = msg;
      }
      s.filling = false;
      f.cv_done.notify_all();
    }
  }
};

namespace {

int check_pool_args(const size_t* layer_off, const size_t* layer_bytes, int n_layers, int depth, void* slots_dev,
                    size_t slot_bytes, size_t off_align, const char* who) {
  if (!layer_off || !layer_bytes || !slots_dev) return fail(NF4LS_INVALID_ARG, "%s: null pointer", who);
  if (n_layers <= 0) return fail(NF4LS_INVALID_ARG, "%s: n_layers must be positive", who);
  if (depth < 2 || depth > 8) return fail(NF4LS_INVALID_ARG, "%s: depth %d not in [2, 8]", who, depth);
  if (!aligned(slots_dev, 256) || slot_bytes % 256)
    return fail(NF4LS_ALIGN, "%s: slots must be 256-byte aligned and sized", who);
  for (int i = 0; i < n_layers; ++i) {
    if (layer_bytes[i] > slot_bytes)
      return fail(NF4LS_INVALID_ARG, "%s: layer %d (%zu B) exceeds slot (%zu B)", who, i, layer_bytes[i], slot_bytes);
    if (layer_off[i] % off_align) return fail(NF4LS_ALIGN, "%s: layer %d offset not %zu-aligned", who, i, off_align);
  }
  return NF4LS_OK;
}

int make_pool(const size_t* layer_off, const size_t* layer_bytes, int n_layers, int depth, void* slots_dev,
              size_t slot_bytes, nf4ls_pool** out) {
  nf4ls_pool* p = new nf4ls_pool();
  p->off.assign(layer_off, layer_off + n_layers);
  p->bytes.assign(layer_bytes, layer_bytes + n_layers);
  p->n_layers = n_layers;
  p->depth = depth;
  p->slots = static_cast<uint8_t*>(slots_dev);
  p->slot_bytes = slot_bytes;
  p->slot.resize(depth);
  p->plan.init(n_layers, depth);
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->copy, cudaStreamNonBlocking);
  for (int i = 0; i < depth && e == cudaSuccess; ++i) {
    e = cudaEventCreateWithFlags(&p->slot[i].ready, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->slot[i].freed, cudaEventDisableTiming);
  }
  if (e != cudaSuccess) {
    nf4ls_pool_destroy(p);
    return fail(NF4LS_CUDA, "pool create: %s", cudaGetErrorString(e));
  }
  *out = p;
  return NF4LS_OK;
}

// sysfs path of the block device holding st_dev, or "" (not a block device).
std::string block_sysfs(dev_t dev) {
  char link[64], real[PATH_MAX];
  std::snprintf(link, sizeof(link), "/sys/dev/block/%u:%u", major(dev), minor(dev));
  if (!realpath(link, real)) return "";
  return real;
}

int read_flag(const std::string& path, int* v) {
  FILE* f = std::fopen(path.c_str(), "r");
  if (!f) return -1;
  const int n = std::fscanf(f, "%d", v);
  std::fclose(f);
  return n == 1 ? 0 : -1;
}

}  // namespace

extern "C" int nf4ls_pool_create(const void* pinned_host, const size_t* layer_off, const size_t* layer_bytes,
                                 int n_layers, int depth, void* slots_dev, size_t slot_bytes, nf4ls_pool** out) {
  clear_error();
  if (!pinned_host || !out) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_create: null pointer");
  NF4_TRY(check_pool_args(layer_off, layer_bytes, n_layers, depth, slots_dev, slot_bytes, 256, "nf4ls_pool_create"));
  NF4_TRY(make_pool(layer_off, layer_bytes, n_layers, depth, slots_dev, slot_bytes, out));
  (*out)->store = static_cast<const uint8_t*>(pinned_host);
  return NF4LS_OK;
}

extern "C" size_t nf4ls_pool_file_staging_bytes(const size_t* layer_bytes, int n_layers) {
  if (!layer_bytes || n_layers <= 0) return 0;
  size_t mx = 0;
  for (int i = 0; i < n_layers; ++i) mx = std::max(mx, layer_bytes[i]);
  return 2 * io_round(mx);
}

extern "C" int nf4ls_pool_create_file(const char* path, const size_t* layer_off, const size_t* layer_bytes,
                                      int n_layers, int depth, void* slots_dev, size_t slot_bytes,
                                      void* staging_host, size_t staging_bytes, nf4ls_pool** out) {
  clear_error();
  if (!path || !staging_host || !out) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_create_file: null pointer");
  NF4_TRY(check_pool_args(layer_off, layer_bytes, n_layers, depth, slots_dev, slot_bytes, kIoAlign,
                          "nf4ls_pool_create_file"));
  const size_t need = nf4ls_pool_file_staging_bytes(layer_bytes, n_layers);
  if (!aligned(staging_host, kIoAlign) || staging_bytes < need)
    return fail(NF4LS_ALIGN, "nf4ls_pool_create_file: staging must be 4096-byte aligned and >= %zu B", need);
  int fd = open(path, O_RDONLY | O_DIRECT);
  bool direct = fd >= 0;
  if (fd < 0) fd = open(path, O_RDONLY);
  if (fd < 0) return fail(NF4LS_IO, "nf4ls_pool_create_file: cannot open %s: %s", path, strerror(errno));
  struct stat st;
  if (fstat(fd, &st) != 0) {
    close(fd);
    return fail(NF4LS_IO, "nf4ls_pool_create_file: fstat failed");
  }
  for (int i = 0; i < n_layers; ++i)
    if (layer_off[i] + layer_bytes[i] > (size_t)st.st_size) {
      close(fd);
      return fail(NF4LS_INVALID_ARG, "nf4ls_pool_create_file: layer %d ends past the end of %s", i, path);
    }
  nf4ls_pool* p = nullptr;
  const int r = make_pool(layer_off, layer_bytes, n_layers, depth, slots_dev, slot_bytes, &p);
  if (r) {
    close(fd);
    return r;
  }
  FileSource* f = new FileSource();
  f->fd = fd;
  f->direct = direct;
  f->staging_each = need / 2;
  f->staging[0] = static_cast<uint8_t*>(staging_host);
  f->staging[1] = f->staging[0] + f->staging_each;
  cudaError_t e = cudaEventCreateWithFlags(&f->staged[0], cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&f->staged[1], cudaEventDisableTiming);
  p->file = f;
  if (e != cudaSuccess) {
    nf4ls_pool_destroy(p);
    return fail(NF4LS_CUDA, "nf4ls_pool_create_file: %s", cudaGetErrorString(e));
  }
  f->reader = std::thread([p] { p->reader_loop(); });
  *out = p;
  return NF4LS_OK;
}

extern "C" int nf4ls_nccl_unique_id(uint8_t id_out[128]) {
  clear_error();
  if (!id_out) return fail(NF4LS_INVALID_ARG, "nf4ls_nccl_unique_id: null output");
  const NcclApi& n = nccl_api();
  if (!n.ok) return fail(NF4LS_CUDA, "nf4ls_nccl_unique_id: libnccl.so.2 not found");
  ncclUniqueId id;
  const ncclResult_t r = n.get_unique_id(&id);
  if (r != ncclSuccess) return fail(NF4LS_CUDA, "ncclGetUniqueId: %s", n.error_string(r));
  static_assert(sizeof(id) == 128, "NCCL unique id size");
  std::memcpy(id_out, &id, sizeof(id));
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_share(nf4ls_pool* p, int rank, int world, const uint8_t id[128]) {
  clear_error();
  if (!p || !id || world < 1 || rank < 0 || rank >= world)
    return fail(NF4LS_INVALID_ARG, "nf4ls_pool_share: bad argument (rank %d, world %d)", rank, world);
  std::lock_guard<std::mutex> g(p->mu);
  if (p->file) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_share: a pool with a file store cannot be shared");
  if (p->comm) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_share: already shared");
  if (p->plan.holds_any()) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_share: the pool must not hold a layer yet");
  const NcclApi& n = nccl_api();
  if (!n.ok) return fail(NF4LS_CUDA, "nf4ls_pool_share: libnccl.so.2 not found");
  NF4_CUDA_TRY(cudaSetDevice(p->device));
  ncclUniqueId uid;
  std::memcpy(&uid, id, sizeof(uid));
  ncclComm_t comm = nullptr;
  const ncclResult_t r = n.comm_init_rank(&comm, world, uid, rank);
  if (r != ncclSuccess) return fail(NF4LS_CUDA, "ncclCommInitRank: %s", n.error_string(r));
  p->comm = comm;
  p->rank = rank;
  p->world = world;
  p->plan.share(rank, world);
  return NF4LS_OK;
}

extern "C" int nf4ls_disk_probe(const char* path, size_t probe_bytes, nf4ls_disk_info* out) {
  clear_error();
  if (!path || !out || probe_bytes == 0) return fail(NF4LS_INVALID_ARG, "nf4ls_disk_probe: bad argument");
  std::memset(out, 0, sizeof(*out));
  struct stat st;
  if (stat(path, &st) != 0) return fail(NF4LS_IO, "nf4ls_disk_probe: cannot stat %s: %s", path, strerror(errno));
  const std::string sys = block_sysfs(st.st_dev);
  if (!sys.empty()) {
    out->block_device = 1;
    out->nvme = sys.find("/nvme") != std::string::npos ? 1 : 0;
    int rot = 0;
    if (read_flag(sys + "/queue/rotational", &rot) != 0) read_flag(sys + "/../queue/rotational", &rot);
    out->rotational = rot ? 1 : 0;
  }
  int fd = open(path, O_RDONLY | O_DIRECT);
  out->direct_io = fd >= 0;
  if (fd < 0) {
    fd = open(path, O_RDONLY);
    if (fd >= 0) posix_fadvise(fd, 0, 0, POSIX_FADV_DONTNEED);  // best effort: start cold
  }
  if (fd < 0) return fail(NF4LS_IO, "nf4ls_disk_probe: cannot open %s: %s", path, strerror(errno));
  const size_t chunk = 16u << 20;
  void* buf = nullptr;
  if (posix_memalign(&buf, kIoAlign, chunk) != 0) {
    close(fd);
    return fail(NF4LS_INVALID_ARG, "nf4ls_disk_probe: no host memory for the probe buffer");
  }
  const size_t total = std::min(probe_bytes, (size_t)st.st_size);
  size_t done = 0;
  int err = 0;
  const auto t0 = std::chrono::steady_clock::now();
  while (done < total) {
    const ssize_t r = pread(fd, buf, chunk, (off_t)done);
    if (r < 0) {
      if (errno == EINTR) continue;
      err = errno;
      break;
    }
    if (r == 0) break;
    done += (size_t)r;
  }
  const double secs = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
  std::free(buf);
  close(fd);
  if (err) return fail(NF4LS_IO, "nf4ls_disk_probe: read failed: %s", strerror(err));
  out->read_gbs = secs > 0 ? (double)done / secs / 1e9 : 0.0;
  return NF4LS_OK;
}

extern "C" int nf4ls_disk_accept(const nf4ls_disk_info* info, double min_gbs) {
  clear_error();
  if (!info) return fail(NF4LS_INVALID_ARG, "nf4ls_disk_accept: null info");
  if (info->rotational) return fail(NF4LS_SOURCE_REFUSED, "stream source refused: spinning disk");
  if (info->block_device && !info->nvme) return fail(NF4LS_SOURCE_REFUSED, "stream source refused: not an NVMe device");
  if (info->read_gbs < min_gbs)
    return fail(NF4LS_SOURCE_REFUSED, "stream source refused: reads at %.2f GB/s < %.2f GB/s", info->read_gbs, min_gbs);
  return NF4LS_OK;
}

extern "C" int nf4ls_choose_source(size_t store_bytes, size_t reserve_bytes, int32_t* use_disk) {
  clear_error();
  if (!use_disk) return fail(NF4LS_INVALID_ARG, "nf4ls_choose_source: null output");
  *use_disk = 0;
  FILE* f = std::fopen("/proc/meminfo", "r");
  if (!f) return NF4LS_OK;  // unknown: memory
  char key[64];
  unsigned long long kb = 0;
  bool found = false;
  while (std::fscanf(f, "%63s %llu kB\n", key, &kb) == 2) {
    if (std::strcmp(key, "MemAvailable:") == 0) {
      found = true;
      break;
    }
  }
  std::fclose(f);
  if (found && (unsigned long long)(store_bytes + reserve_bytes) > kb * 1024ull) *use_disk = 1;
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_prefetch(nf4ls_pool* p, int layer) {
  clear_error();
  if (!p || layer < 0 || layer >= p->n_layers) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_prefetch: bad argument");
  std::lock_guard<std::mutex> g(p->mu);
  int idx;
  return p->issue(layer, &idx);
}

extern "C" int stream_prefetch(nf4ls_pool* p, int layer, nf4ls_stream compute, const void** slot_dev) {
  clear_error();
  if (!p || layer < 0 || layer >= p->n_layers || !slot_dev)
    return fail(NF4LS_INVALID_ARG, "stream_prefetch: bad argument");
  std::unique_lock<std::mutex> lk(p->mu);
  const bool hit = p->find(layer) >= 0;  // resident or already prefetched: this call copies nothing
  int idx;
  NF4_TRY(p->issue(layer, &idx));
  nf4ls_pool::Slot& s = p->slot[idx];
  if (p->plan.acquired(idx)) return fail(NF4LS_BUFFER_BUSY, "stream_prefetch: layer %d is already acquired", layer);
  NF4_TRY(p->wait_filled(lk, idx));
  NF4_CUDA_TRY(cudaStreamWaitEvent(static_cast<cudaStream_t>(compute), s.ready, 0));
  p->plan.mark_acquired(idx);
  p->stats.acquisitions += 1;
  if (hit) p->stats.hits += 1;
  *slot_dev = p->slots + (size_t)idx * p->slot_bytes;
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_release(nf4ls_pool* p, int layer, nf4ls_stream compute) {
  clear_error();
  if (!p || layer < 0 || layer >= p->n_layers) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_release: bad argument");
  std::lock_guard<std::mutex> g(p->mu);
  const int idx = p->plan.acquired_slot(layer);
  if (idx < 0) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_release: layer %d not acquired", layer);
  NF4_CUDA_TRY(cudaEventRecord(p->slot[idx].freed, static_cast<cudaStream_t>(compute)));
  p->plan.release(idx);
  return NF4LS_OK;
}

extern "C" int nf4ls_wait(nf4ls_pool* p, int layer, int timeout_ms) {
  clear_error();
  if (!p || layer < 0 || layer >= p->n_layers) return fail(NF4LS_INVALID_ARG, "nf4ls_wait: bad argument");
  cudaEvent_t ev;
  {
    std::unique_lock<std::mutex> lk(p->mu);
    const int idx = p->find(layer);
    if (idx < 0) return fail(NF4LS_INVALID_ARG, "nf4ls_wait: layer %d has no slot", layer);
    NF4_TRY(p->wait_filled(lk, idx));
    ev = p->slot[idx].ready;
  }
  const auto t0 = std::chrono::steady_clock::now();
  while (true) {
    const cudaError_t e = cudaEventQuery(ev);
    if (e == cudaSuccess) return NF4LS_OK;
    if (e != cudaErrorNotReady) return fail(NF4LS_CUDA, "nf4ls_wait: %s", cudaGetErrorString(e));
    const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0);
    if (ms.count() >= timeout_ms) return fail(NF4LS_TIMEOUT, "nf4ls_wait: layer %d not ready after %d ms", layer, timeout_ms);
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
}

extern "C" int nf4ls_pool_set_poison(nf4ls_pool* p, int on) {
  if (!p) return fail(NF4LS_INVALID_ARG, "null pool");
  std::lock_guard<std::mutex> g(p->mu);
  p->poison = on != 0;
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_get_stats(nf4ls_pool* p, nf4ls_pool_stats* out) {
  if (!p || !out) return fail(NF4LS_INVALID_ARG, "null argument");
  std::lock_guard<std::mutex> g(p->mu);
  *out = p->stats;
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_synchronize(nf4ls_pool* p) {
  if (!p) return fail(NF4LS_INVALID_ARG, "null pool");
  if (p->file) {
    std::unique_lock<std::mutex> lk(p->mu);
    p->file->cv_done.wait_for(lk, std::chrono::milliseconds(kFillWaitMs),
                              [&] { return p->file->jobs.empty() || p->file->error != NF4LS_OK; });
    if (p->file->error) return fail(p->file->error, "pool: disk source: %s", p->file->error_msg.c_str());
  }
  NF4_CUDA_TRY(cudaStreamSynchronize(p->copy));
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_destroy(nf4ls_pool* p) {
  if (!p) return NF4LS_OK;
  if (p->file) {
    {
      std::lock_guard<std::mutex> g(p->mu);
      p->file->stop = true;
      p->file->cv_job.notify_all();
    }
    if (p->file->reader.joinable()) p->file->reader.join();
  }
  if (p->copy) cudaStreamSynchronize(p->copy);
  if (p->comm) nccl_api().comm_destroy(p->comm);
  if (p->file) {
    for (int b = 0; b < 2; ++b)
      if (p->file->staged[b]) cudaEventDestroy(p->file->staged[b]);
    if (p->file->fd >= 0) close(p->file->fd);
    delete p->file;
    p->file = nullptr;
  }
  for (auto& s : p->slot) {
    if (s.ready) cudaEventDestroy(s.ready);
    if (s.freed) cudaEventDestroy(s.freed);
  }
  if (p->copy) cudaStreamDestroy(p->copy);
  delete p;
  return NF4LS_OK;
}
