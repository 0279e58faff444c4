// TapChannel: a side channel that carries target features from producer
// pipeline stages to the stage holding the draft, outside the pipeline's own
// schedule ("Online Draft Co-Training", method-detail section, pipeline
// transport item; technical-contribution section: mailboxes, sequence stamps
// and pre-allocated slots, CUDA IPC within a node).
//
// The consumer owns one device region, the mailbox:
//   stamps [P][S] int64   written by producer p once slot s holds message seq
//   acks   [P][S] int64   written by the consumer once it is done with slot s
//   slots  [P][S][slot_bytes]
// and shares it with the producers through a CUDA IPC handle.  Message seq of
// producer p goes to slot seq mod S.
//   send (producer): wait on the host until ack[p][s] >= seq - S (the slot's
//     previous message has been released), copy the payload into the slot with
//     the copy engine (over NVLink when the consumer is another GPU), then a
//     one-thread kernel on the same stream writes stamp[p][s] = seq.  Stream
//     order puts the stamp after the payload.
//   wait (consumer): poll stamp[p][s] on the host until it equals seq; the
//     payload is then complete in the consumer's memory.
//   release (consumer): a one-thread kernel on the consumer's stream writes
//     ack[p][s] = seq after the work that read the slot.
// No kernel waits on another process: every wait is a bounded host poll, so
// producers and consumer may even share one GPU.
#include <chrono>
#include <cstring>
#include <thread>

#include "internal.cuh"

namespace ba {
namespace {

constexpr uint64_t kTapMagic = 0x7a70436c61746e54ull;  // identifies a handle blob

struct TapHandleBlob {
  uint64_t magic;
  int32_t n_producers, n_slots;
  int64_t slot_bytes;
  uint64_t offset;  // the mailbox's offset inside the allocation the handle names
  cudaIpcMemHandle_t mem;
};

static_assert(sizeof(TapHandleBlob) <= 128, "the handle blob must fit the documented 128 bytes");

using AddressRangeFn = int (*)(unsigned long long *, size_t *, unsigned long long);

// The driver's cuMemGetAddressRange, found through the runtime (the library
// links no driver library); null if unavailable.
AddressRangeFn address_range() {
  static AddressRangeFn fn = nullptr;
  static bool looked = false;
  if (!looked) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(p);
    looked = true;
  }
  return fn;
}

__global__ void tap_store_kernel(volatile long long *word, long long value) {
  __threadfence_system();
  *word = value;
  __threadfence_system();
}

size_t header_bytes(int32_t p, int32_t s) {
  const size_t words = (size_t)2 * p * s * 8;
  return (words + 255) / 256 * 256;
}

}  // namespace
}  // namespace ba

using namespace ba;

struct ba_tap {
  int32_t n_producers, n_slots, producer;  // producer = -1 on the consumer side
  int64_t slot_bytes;
  char *base;       // mailbox (own memory for the consumer, IPC mapping for a producer)
  void *ipc_base;   // what cudaIpcOpenMemHandle returned (producer side)
  bool mapped;      // opened through cudaIpcOpenMemHandle
  int device;
};

namespace {

ba_status check_dims(int32_t p, int32_t s, int64_t b) {
  if (p < 1 || p > 256 || s < 1 || s > 1024 || b < 16 || b % 16 != 0) {
    set_error("tap: need 1 <= producers <= 256, 1 <= slots <= 1024, slot bytes a positive "
              "multiple of 16 (got %d, %d, %lld)", p, s, (long long)b);
    return BA_ERR_INVALID_ARG;
  }
  return BA_OK;
}

long long *stamp_word(const ba_tap *t, int32_t p, int32_t s) {
  return reinterpret_cast<long long *>(t->base) + (size_t)p * t->n_slots + s;
}
long long *ack_word(const ba_tap *t, int32_t p, int32_t s) {
  return reinterpret_cast<long long *>(t->base) + (size_t)t->n_producers * t->n_slots +
         (size_t)p * t->n_slots + s;
}
char *slot_ptr(const ba_tap *t, int32_t p, int32_t s) {
  return t->base + header_bytes(t->n_producers, t->n_slots) +
         ((size_t)p * t->n_slots + s) * (size_t)t->slot_bytes;
}

// Reads one 8-byte word of (possibly peer) device memory from the host.
ba_status read_word(const long long *word, long long *out) {
  return cuda_check(cudaMemcpy(out, word, 8, cudaMemcpyDeviceToHost), "tap: read stamp");
}

// Polls until pred(word) holds or timeout_ns passes.
template <typename Pred>
ba_status poll_word(const long long *word, int64_t timeout_ns, Pred pred, const char *what) {
  const auto t0 = std::chrono::steady_clock::now();
  for (int i = 0;; ++i) {
    long long v = 0;
    ba_status st = read_word(word, &v);
    if (st != BA_OK) return st;
    if (pred(v)) return BA_OK;
    const int64_t el = std::chrono::duration_cast<std::chrono::nanoseconds>(
                           std::chrono::steady_clock::now() - t0).count();
    if (el > timeout_ns) {
      set_error("tap: timed out after %lld ns waiting for %s (last value %lld)",
                (long long)el, what, v);
      return BA_ERR_DEVICE_TIMEOUT;
    }
    if (i > 64) std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

ba_status store_word(long long *word, long long value, cudaStream_t s) {
  tap_store_kernel<<<1, 1, 0, s>>>(word, value);
  count_launches(1);
  return cuda_check(cudaGetLastError(), "tap: stamp kernel");
}

}  // namespace

extern "C" {

ba_status ba_tap_mailbox_size(int32_t n_producers, int32_t n_slots, int64_t slot_bytes,
                              size_t *bytes) {
  ba_status st = check_dims(n_producers, n_slots, slot_bytes);
  if (st != BA_OK) return st;
  if (!bytes) {
    set_error("tap: bytes is NULL");
    return BA_ERR_INVALID_ARG;
  }
  *bytes = header_bytes(n_producers, n_slots) +
           (size_t)n_producers * n_slots * (size_t)slot_bytes;
  return BA_OK;
}

ba_status ba_tap_create(void *mailbox, size_t mailbox_bytes, int32_t n_producers,
                        int32_t n_slots, int64_t slot_bytes, void *handle_out,
                        size_t handle_bytes, ba_tap **out) {
  size_t need = 0;
  ba_status st = ba_tap_mailbox_size(n_producers, n_slots, slot_bytes, &need);
  if (st != BA_OK) return st;
  if (!mailbox || !out || !handle_out) {
    set_error("tap: mailbox, handle_out and out are required");
    return BA_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(mailbox) % 256 != 0) {
    set_error("tap: the mailbox must be 256-byte aligned");
    return BA_ERR_MISALIGNED;
  }
  if (mailbox_bytes < need) {
    set_error("tap: mailbox too small: %zu < %zu bytes", mailbox_bytes, need);
    return BA_ERR_WORKSPACE_TOO_SMALL;
  }
  if (handle_bytes < sizeof(TapHandleBlob)) {
    set_error("tap: handle buffer too small: %zu < %zu bytes", handle_bytes,
              sizeof(TapHandleBlob));
    return BA_ERR_WORKSPACE_TOO_SMALL;
  }
  TapHandleBlob blob;
  std::memset(&blob, 0, sizeof(blob));
  blob.magic = kTapMagic;
  blob.n_producers = n_producers;
  blob.n_slots = n_slots;
  blob.slot_bytes = slot_bytes;
  // the IPC handle names the whole allocation that holds the mailbox (a
  // caching allocator hands out pieces of larger blocks): record where in it
  // the mailbox starts
  AddressRangeFn range = address_range();
  unsigned long long alloc_base = 0;
  size_t alloc_size = 0;
  if (!range || range(&alloc_base, &alloc_size, reinterpret_cast<unsigned long long>(mailbox)) != 0) {
    set_error("tap: cannot find the allocation that holds the mailbox");
    return BA_ERR_CUDA;
  }
  blob.offset = reinterpret_cast<unsigned long long>(mailbox) - alloc_base;
  if (blob.offset + need > alloc_size) {
    set_error("tap: the mailbox runs past the end of its allocation");
    return BA_ERR_INVALID_ARG;
  }
  st = cuda_check(cudaIpcGetMemHandle(&blob.mem, mailbox), "tap: cudaIpcGetMemHandle");
  if (st != BA_OK) return st;
  // stamps and acks start at -1 (no message), written before any producer attaches
  st = cuda_check(cudaMemset(mailbox, 0xff, header_bytes(n_producers, n_slots)),
                  "tap: clearing stamps");
  if (st != BA_OK) return st;
  st = cuda_check(cudaDeviceSynchronize(), "tap: clearing stamps");
  if (st != BA_OK) return st;
  ba_tap *t = new ba_tap;
  t->n_producers = n_producers;
  t->n_slots = n_slots;
  t->producer = -1;
  t->slot_bytes = slot_bytes;
  t->base = reinterpret_cast<char *>(mailbox);
  t->ipc_base = nullptr;
  t->mapped = false;
  cudaGetDevice(&t->device);
  std::memcpy(handle_out, &blob, sizeof(blob));
  *out = t;
  return BA_OK;
}

ba_status ba_tap_attach(const void *handle, size_t handle_bytes, int32_t producer,
                        ba_tap **out) {
  if (!handle || !out || handle_bytes < sizeof(TapHandleBlob)) {
    set_error("tap: a handle of %zu bytes and out are required", sizeof(TapHandleBlob));
    return BA_ERR_INVALID_ARG;
  }
  TapHandleBlob blob;
  std::memcpy(&blob, handle, sizeof(blob));
  if (blob.magic != kTapMagic) {
    set_error("tap: not a mailbox handle");
    return BA_ERR_INVALID_ARG;
  }
  ba_status st = check_dims(blob.n_producers, blob.n_slots, blob.slot_bytes);
  if (st != BA_OK) return st;
  if (producer < 0 || producer >= blob.n_producers) {
    set_error("tap: producer %d outside [0, %d)", producer, blob.n_producers);
    return BA_ERR_INVALID_ARG;
  }
  void *p = nullptr;
  st = cuda_check(cudaIpcOpenMemHandle(&p, blob.mem, cudaIpcMemLazyEnablePeerAccess),
                  "tap: cudaIpcOpenMemHandle");
  if (st != BA_OK) return st;
  ba_tap *t = new ba_tap;
  t->n_producers = blob.n_producers;
  t->n_slots = blob.n_slots;
  t->producer = producer;
  t->slot_bytes = blob.slot_bytes;
  t->base = reinterpret_cast<char *>(p) + blob.offset;
  t->ipc_base = p;
  t->mapped = true;
  cudaGetDevice(&t->device);
  *out = t;
  return BA_OK;
}

ba_status ba_tap_send(ba_tap *t, int64_t seq, const void *src, int64_t bytes,
                      int64_t timeout_ns, ba_stream_t stream) {
  if (!t || t->producer < 0) {
    set_error("tap: send needs a producer-side channel");
    return BA_ERR_INVALID_ARG;
  }
  if (seq < 0 || !src || bytes < 0 || bytes > t->slot_bytes) {
    set_error("tap: need seq >= 0, a source and 0 <= bytes <= slot bytes %lld (got %lld)",
              (long long)t->slot_bytes, (long long)bytes);
    return BA_ERR_INVALID_ARG;
  }
  const int32_t s = (int32_t)(seq % t->n_slots);
  // the slot's previous message (seq - S) must have been released
  const long long need = seq - t->n_slots;
  ba_status st = poll_word(ack_word(t, t->producer, s), timeout_ns,
                           [need](long long v) { return v >= need; }, "a free slot");
  if (st != BA_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  if (bytes > 0) {
    st = cuda_check(cudaMemcpyAsync(slot_ptr(t, t->producer, s), src, (size_t)bytes,
                                    cudaMemcpyDeviceToDevice, cs),
                    "tap: payload copy");
    if (st != BA_OK) return st;
  }
  return store_word(stamp_word(t, t->producer, s), seq, cs);
}

ba_status ba_tap_wait(ba_tap *t, int32_t producer, int64_t seq, int64_t timeout_ns,
                      void **slot) {
  if (!t || t->producer >= 0) {
    set_error("tap: wait needs the consumer-side channel");
    return BA_ERR_INVALID_ARG;
  }
  if (producer < 0 || producer >= t->n_producers || seq < 0) {
    set_error("tap: producer %d outside [0, %d) or negative seq", producer, t->n_producers);
    return BA_ERR_INVALID_ARG;
  }
  const int32_t s = (int32_t)(seq % t->n_slots);
  ba_status st = poll_word(stamp_word(t, producer, s), timeout_ns,
                           [seq](long long v) { return v == seq; }, "a message stamp");
  if (st != BA_OK) return st;
  if (slot) *slot = slot_ptr(t, producer, s);
  return BA_OK;
}

ba_status ba_tap_release(ba_tap *t, int32_t producer, int64_t seq, ba_stream_t stream) {
  if (!t || t->producer >= 0) {
    set_error("tap: release needs the consumer-side channel");
    return BA_ERR_INVALID_ARG;
  }
  if (producer < 0 || producer >= t->n_producers || seq < 0) {
    set_error("tap: producer %d outside [0, %d) or negative seq", producer, t->n_producers);
    return BA_ERR_INVALID_ARG;
  }
  return store_word(ack_word(t, producer, (int32_t)(seq % t->n_slots)), seq,
                    (cudaStream_t)stream);
}

ba_status ba_tap_close(ba_tap *t) {
  if (!t) return BA_OK;
  ba_status st = BA_OK;
  if (t->mapped) st = cuda_check(cudaIpcCloseMemHandle(t->ipc_base), "tap: cudaIpcCloseMemHandle");
  delete t;
  return st;
}

}  // extern "C"
