// mbok_gemv_noalloc: the decode GEMV for callers that cannot allocate device
// memory.  Its scratch (the per-slab partial sums that mbok_gemv keeps in a
// caller-provided workspace) lives in a fixed-size array compiled into this
// library instead.  The library allocates nothing here.
#include "mbok_common.cuh"

namespace mbok {
cudaError_t launch_gemv(const uint8_t*, const uint16_t*, const Shape&, const void*, bool, int, float*,
                        void*, cudaStream_t);
cudaError_t launch_gemv_lut(const uint8_t*, const uint16_t*, const Shape&, const void*, bool,
                            float*, void*, cudaStream_t, bool);
size_t gemv_lut_workspace_bytes(const Shape&);
}  // namespace mbok

using namespace mbok;

// The scratch array.  Every GPU that loads the library holds it until the
// process exits.  In host code `g_noalloc_scratch` names a host-side stand-in,
// not the device array, so host code only ever passes the device address
// obtained from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MBOK_NOALLOC_SCRATCH_BYTES];

namespace {

// Set-up, once per device, with that device current: the device address of
// the scratch array (cached per device index; host threads making their
// first calls together at worst both look it up).  nullptr if the runtime
// refuses.
void* scratch_address() {
  static PerDeviceValue<void*> cache;
  const int dev = current_device();
  if (dev < 0) return nullptr;
  return cache.get(dev, []() -> void* {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    return ptr;
  });
}

}  // namespace

extern "C" int mbok_gemv_noalloc(const uint32_t* packed, const uint16_t* alpha, int K, int M,
                                 int N, int group, const void* x, int x_dtype, int batch, float* y,
                                 void* stream) {
  if (K < 1 || K > MBOK_MAX_K) return MBOK_ERR_INVALID_ARG;
  if (M < 1 || N < MBOK_GROUP || N % MBOK_GROUP != 0 || M > (1 << 22) || N > (1 << 20))
    return MBOK_ERR_SHAPE;
  if (group != MBOK_GROUP) return MBOK_ERR_UNSUPPORTED;
  if (packed == nullptr || alpha == nullptr || x == nullptr || y == nullptr)
    return MBOK_ERR_INVALID_ARG;
  if (x_dtype != MBOK_F32 && x_dtype != MBOK_BF16) return MBOK_ERR_INVALID_ARG;
  if (batch < 1 || batch > MBOK_MAX_BATCH) return MBOK_ERR_INVALID_ARG;
  const uintptr_t a16 = 15;
  if ((reinterpret_cast<uintptr_t>(packed) & a16) || (reinterpret_cast<uintptr_t>(alpha) & a16) ||
      (reinterpret_cast<uintptr_t>(x) & a16) || (reinterpret_cast<uintptr_t>(y) & 3))
    return MBOK_ERR_ALIGN;
  const Shape s = make_shape(K, M, N);
  const size_t need = gemv_lut_workspace_bytes(s);
  if (need > size_t(MBOK_NOALLOC_SCRATCH_BYTES)) return MBOK_ERR_SCRATCH_LIMIT;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  if (need > 0) {
    scratch = scratch_address();
    if (scratch == nullptr) return MBOK_ERR_CUDA;
  }
  if (launch_gemv(reinterpret_cast<const uint8_t*>(packed), alpha, s, x, x_dtype == MBOK_F32, batch, y,
                  scratch, st) != cudaSuccess)
    return MBOK_ERR_CUDA;
  return MBOK_OK;
}
