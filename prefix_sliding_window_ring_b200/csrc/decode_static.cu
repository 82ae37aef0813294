// Decode attention for callers that cannot allocate device memory.
//
// ps_attend_decode needs a caller-provided workspace for its split-K partial
// results.  Some callers cannot provide one: a host runtime that owns every
// byte of device memory through its own pool and gives plug-ins no way to ask
// for more, or a latency-critical serving loop in which a cudaMalloc (which
// synchronises the whole device) is not acceptable.  ps_attend_decode_static
// runs the same decode kernel with its scratch in a fixed-size array that is
// part of this library's device image, so it allocates nothing.
//
// The array is file-scope device memory: every GPU that loads the library
// holds kStaticScratchBytes of it until the process exits, and all calls on a
// device share it.  In host code the array's name only stands for the symbol;
// its device address comes from cudaGetSymbolAddress, looked up once per
// device (with that device current) on the first call and cached.
#include <mutex>

#include "ps.h"
#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)4 << 20;  // 4 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The first call
// on a device looks the address up and zero-fills the array (the decode keeps
// no state in it between calls; the fill only gives it defined contents).
// That set-up synchronises the device, so the first call on each device must
// not be made while a stream is being captured.
cudaError_t scratch_on_current_device(void** out, int* dev_out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  *dev_out = dev;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    e = cudaMemset(p, 0, kStaticScratchBytes);
    if (e != cudaSuccess) return e;
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

int ps_attend_decode_static(ps_cache* c, const void* q, const int* seq_ids, const int64_t* t,
                            int B, int Hq, float scale, void* out, void* stream) {
  if (!c) return ps::set_error(PS_EINVAL, "ps_attend_decode_static: cache is NULL");
  if (B < 0 || Hq < 1) return ps::set_error(PS_EINVAL, "ps_attend_decode_static: bad B or Hq");
  if (B > 0 && (!seq_ids || !t))
    return ps::set_error(PS_EINVAL, "ps_attend_decode_static: seq_ids/t is NULL");
  // Scratch this call needs: the same layout ps_attend_decode uses.
  const int Hkv = ps::cache_hkv(c);
  if (Hq % Hkv) return ps_attend_decode(c, q, seq_ids, t, B, Hq, scale, out, nullptr, 0, stream);
  size_t need = 0;
  ps::decode_ws_layout(nullptr, B, Hkv, Hq / Hkv, ps::cache_head_dim(c), ps::cache_sm_count(c),
                       &need);
  if (need > kStaticScratchBytes)
    return ps::set_error(PS_ENOMEM,
                         "ps_attend_decode_static: this batch needs %zu bytes of scratch, above "
                         "the fixed %zu-byte array; use ps_attend_decode with a workspace",
                         need, kStaticScratchBytes);
  void* scratch = nullptr;
  int dev = -1;
  cudaError_t e = scratch_on_current_device(&scratch, &dev);
  if (e != cudaSuccess)
    return ps::set_error(PS_ECUDA, "ps_attend_decode_static: scratch set-up on device %d: %s",
                         dev, cudaGetErrorString(e));
  return ps_attend_decode(c, q, seq_ids, t, B, Hq, scale, out, scratch, kStaticScratchBytes,
                          stream);
}

}  // extern "C"
