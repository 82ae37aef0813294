// Decode attention for callers that cannot allocate device memory.
//
// ps_attend_decode needs a caller-provided workspace for its split-K partial
// results.  Some callers cannot provide one: a host runtime that owns every
// byte of device memory through its own pool and gives plug-ins no way to ask
// for more, or a latency-critical serving loop in which a cudaMalloc (which
// synchronises the whole device) is not acceptable.  ps_attend_decode_static
// runs the same decode kernels with their scratch in a fixed-size array that
// is part of this library's device image, so it allocates nothing.
//
// The array is file-scope device memory: every GPU that loads the library
// holds kStaticScratchBytes of it until the process exits, and all calls on a
// device share it.  The decode writes every partial it reads in the same call,
// so nothing in the array has to start at zero.  In host code the array's
// name only stands for the symbol; its device address comes from
// cudaGetSymbolAddress, looked up with the device current on the first call
// on that device and cached.  The cache is keyed by the device's context, so
// after a cudaDeviceReset the next call looks the address up again.
#include <cuda.h>

#include <mutex>

#include "ps.h"
#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)4 << 20;  // 4 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

struct ScratchSlot {
  unsigned long long ctx_id;  // context the address belongs to (0: none yet)
  void* ptr;
};

std::mutex g_setup_mutex;
ScratchSlot g_scratch[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if it cannot be read;
// the address is then looked up on every call).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = (CtxGetCurrentFn)p;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = (CtxGetIdFn)p;
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device.  The look-up
// does not synchronise, but it may make the runtime set up the device's
// context and load this library's device code, so the first call on each
// device must not be made while a stream is being captured.
cudaError_t scratch_on_current_device(void** out, int* dev_out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  *dev_out = dev;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  ScratchSlot& s = g_scratch[dev];
  unsigned long long id = current_context_id();
  if (id != 0 && s.ctx_id == id) {  // set up already, in this context
    *out = s.ptr;
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_decode_scratch);  // binds the device's context if needed
  if (e != cudaSuccess) return e;
  s.ctx_id = current_context_id();
  s.ptr = p;
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" {

int ps_attend_decode_static(ps_cache* c, const void* q, const int* seq_ids, const int64_t* t,
                            int B, int Hq, float scale, void* out, void* stream) {
  // Every argument and sequence state is checked before the scratch is set up.
  int G = 0;
  int r = ps::check_decode_call(c, q, seq_ids, t, B, Hq, out, &G);
  if (r) return r;
  if (B == 0) return ps_attend_decode(c, q, seq_ids, t, 0, Hq, scale, out, nullptr, 0, stream);
  // Scratch this call needs: the same layout ps_attend_decode uses.
  size_t need = 0;
  ps::decode_ws_layout(nullptr, B, ps::cache_hkv(c), G, ps::cache_head_dim(c),
                       ps::cache_sm_count(c), &need);
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
