// sage_quantize_noalloc: the smoothing + quantisation stage with its reduction
// scratch (the exact int64 K channel sums, the V channel maxima and a status
// word) held in a fixed, file-scope device array instead of a caller workspace.
//
// Who needs this: code that may not allocate device memory itself and has no
// workspace to hand over -- for example an extension running inside a host
// application that owns every device allocation and only passes it the
// tensors of the call, or a latency-critical path where the implicit device
// synchronisation of cudaMalloc/cudaFree is not acceptable.  Such a caller
// can still provide the stage's inputs and outputs; this entry point needs
// nothing else.
//
// Costs and rules:
//   - The array is SAGE_NOALLOC_SCRATCH_BYTES (1 MiB) of device memory that
//     every GPU which loads the library keeps until the process exits.
//   - It holds the scratch of one call: B*H*D must not exceed
//     SAGE_NOALLOC_MAX_BHD (65536); larger problems are rejected.
//   - All calls share it and it keeps the last call's contents; each call
//     clears the parts that must start at zero.  Calls whose GPU work overlaps
//     (different streams, or several host threads) race on it.
//   - The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current; make that first call
//     before any stream capture.
#include <mutex>

#include "common.cuh"

namespace sage {
cudaError_t launch_quant(const SeqLayout& L, dim3 grid, int D, bool bf16, bool fp8,
                         const void* q, const void* k, const void* v, int8_t* q_codes,
                         float* q_scale, int8_t* k_codes, float* k_scale, float* k_mean,
                         uint8_t* v_codes, float* v_scale, unsigned long long* k_sum,
                         uint32_t* v_amax, uint32_t* status, unsigned int* sync, int parts,
                         int per_token, cudaStream_t st);
}  // namespace sage

namespace {

constexpr size_t kScratchBytes = SAGE_NOALLOC_SCRATCH_BYTES;
constexpr long long kMaxBHD = SAGE_NOALLOC_MAX_BHD;

// Layout: [0, 256) status word; then the int64 K sums; then the V maxima;
// then the work / completion counters of the quantisation kernel (one per
// (batch, head) plus one; B*H <= SAGE_NOALLOC_MAX_BHD / 64).
constexpr size_t kSumOff = 256;
constexpr size_t kAmaxOff = kSumOff + (size_t)kMaxBHD * 8;
constexpr size_t kSyncOff = kAmaxOff + (size_t)kMaxBHD * 4;
constexpr size_t kMaxUnits = kMaxBHD / 64;
static_assert(kSyncOff + (kMaxUnits + 1) * 4 <= kScratchBytes, "scratch layout");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_on_current_device(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_ptr[dev]);
  return cudaSuccess;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" sage_status_t sage_quantize_noalloc(
    const void* q, const void* k, const void* v, int in_dt, int B, int H, int N, int D,
    int pv_mode, int8_t* q_codes, float* q_scale, int8_t* k_codes, float* k_scale,
    float* k_mean, uint8_t* v_codes, float* v_scale, uint32_t* status_out, void* stream) {
  if (B < 1 || H < 1 || N < 1 || N > (1 << 22) || (D != 64 && D != 128) ||
      (in_dt != SAGE_F16 && in_dt != SAGE_BF16) ||
      (pv_mode != SAGE_PV_FP16 && pv_mode != SAGE_PV_FP8) || (long long)B * H > 65535)
    return SAGE_ERR_INVALID_ARG;
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_codes) || !aligned16(k_codes) ||
      !q_scale || !k_scale || !k_mean)
    return SAGE_ERR_INVALID_ARG;
  if (fp8 && (!aligned16(v) || !aligned16(v_codes) || !v_scale)) return SAGE_ERR_INVALID_ARG;
  if ((long long)B * H * D > kMaxBHD) return SAGE_ERR_WORKSPACE;  // beyond the fixed scratch

  unsigned char* scratch = nullptr;
  cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) return SAGE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bhd = (size_t)B * H * D;
  uint32_t* status = status_out ? status_out : reinterpret_cast<uint32_t*>(scratch);
  // the sums and maxima accumulate with atomics: they must start at zero
  e = cudaMemsetAsync(status, 0, sizeof(uint32_t), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(scratch + kSumOff, 0, bhd * 8, st);
  if (e == cudaSuccess && fp8) e = cudaMemsetAsync(scratch + kAmaxOff, 0, bhd * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(scratch + kSyncOff, 0, ((size_t)B * H + 1) * 4, st);
  if (e != cudaSuccess) return SAGE_ERR_CUDA;

  sage::SeqLayout L{};
  L.varlen = 0;
  L.N = N;
  L.H = H;
  e = sage::launch_quant(L, dim3((N + sage::BLK - 1) / sage::BLK, B * H), D, in_dt == SAGE_BF16,
                         fp8, q, k, v, q_codes, q_scale, k_codes, k_scale, k_mean, v_codes,
                         v_scale, reinterpret_cast<unsigned long long*>(scratch + kSumOff),
                         reinterpret_cast<uint32_t*>(scratch + kAmaxOff), status,
                         reinterpret_cast<unsigned int*>(scratch + kSyncOff),
                         sage::QUANT_Q | sage::QUANT_KV, 0, st);
  return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}
