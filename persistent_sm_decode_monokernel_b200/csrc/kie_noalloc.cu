// kie_gemv_f16_noalloc: the weight-stream GEMV engine with every piece of
// device scratch taken from one fixed array compiled into the library,
// for callers that must not allocate device memory.  Who they are: a host
// process that reserved all of the GPU's memory for its own pool at start-up
// (a server that sizes its KV cache to fill HBM), where a cudaMalloc fails
// or takes memory the pool counts on; and a latency-bound loop, where
// cudaMalloc / cudaFree would synchronise the whole device.
//
// The array below is module-scope device memory: every GPU that loads this
// library holds it, once, until the process exits.  Its size bounds the
// matrix (KIE_NOALLOC_MAX_WEIGHT_BYTES of fp16 weights plus a small fixed
// header).  All calls on a device share it and find the last call's
// contents there; whatever must start at zero is cleared on the stream by
// each call.  Two calls whose work overlaps on the GPU (different streams,
// or different host threads) race on it; callers serialise them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <vector>

#include "kie.h"
#include "kie_guard.h"
#include "kie_kernel.h"
#include "kie_params.h"
#include "kie_plan.h"

namespace {

using kie::DevStatus;
using kie::LayerW;
using kie::MonoParams;

constexpr int kMaxCtas = 256;        // more SMs than this: the launch uses 256 CTAs
constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;

constexpr size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// Byte offsets inside the scratch array.
constexpr size_t kOffStatus = 0;
constexpr size_t kOffLayer = round_up(kOffStatus + sizeof(DevStatus));
constexpr size_t kOffRanges = round_up(kOffLayer + sizeof(LayerW));
constexpr size_t kOffPackedOff = round_up(kOffRanges + sizeof(int2) * kie::N_STAGES * kMaxCtas);
constexpr size_t kOffStats = round_up(kOffPackedOff + sizeof(unsigned long long) * kMaxCtas);
constexpr size_t kOffPacked =
    round_up(kOffStats + sizeof(unsigned long long) * kie::kStatsPerCta * kMaxCtas);
constexpr size_t kScratchBytes = kOffPacked + KIE_NOALLOC_MAX_WEIGHT_BYTES;

static_assert(kOffPacked <= 64 * 1024, "scratch header grew past 64 KB");

// The device-side scratch.  In host code this name stands for the symbol,
// not for a device address; the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char kie_noalloc_scratch[kScratchBytes];

std::mutex g_setup_mu;

// Address of the array per device, together with the id of the driver
// context it was looked up in.  A module's device addresses belong to one
// context: after cudaDeviceReset, or with another driver context made
// current on the same device, the array lives at a new address, so a cached
// address is only reused while the current context's id (unique for the
// life of the process) still matches.
struct ScratchAddr {
  unsigned long long ctx_id;
  unsigned char* addr;
};
ScratchAddr g_scratch[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Id of the current driver context; false if the driver cannot tell or no
// context is current yet (then the address is looked up again).
bool current_ctx_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool resolved = false;
  if (!resolved) {
    void* f0 = nullptr;
    void* f1 = nullptr;
    cudaDriverEntryPointQueryResult q0{}, q1{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f0, cudaEnableDefault, &q0) == cudaSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
        q0 == cudaDriverEntryPointSuccess && q1 == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<CtxGetCurrentFn>(f0);
      get_id = reinterpret_cast<CtxGetIdFn>(f1);
    }
    resolved = true;
  }
  CUcontext ctx = nullptr;
  return get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx &&
         get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch in the current device's current context,
// looked up (cudaGetSymbolAddress, which loads the library's device code
// into that context if nothing has yet) on the first call made in that
// context, and reused while the context stays the same.
kie_status scratch_on_current_device(unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return KIE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KIE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  ScratchAddr& e = g_scratch[dev];
  if (!have_id || !e.addr || e.ctx_id != id) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, kie_noalloc_scratch) != cudaSuccess || !ptr)
      return KIE_ERR_CUDA;
    e.addr = static_cast<unsigned char*>(ptr);
    e.ctx_id = have_id ? id : 0ull;
  }
  *out = e.addr;
  return KIE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

kie_status kie_gemv_f16_noalloc(const void* W, const float* x, float* y, int32_t N, int32_t K,
                                void* cuda_stream) {
  return kie::no_throw([&]() -> kie_status {
    constexpr int kChunkBytes = 32768;
    if (!W || !x || !y || N < 1 || K < 256 || K % 256) return KIE_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(x)) return KIE_ERR_INVALID_ARG;
    if ((uint64_t)N * (uint64_t)K * 2u > KIE_NOALLOC_MAX_WEIGHT_BYTES) return KIE_ERR_TOO_LARGE;

    unsigned char* scratch = nullptr;
    kie_status ret = scratch_on_current_device(&scratch);
    if (ret != KIE_OK) return ret;

    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    int dev = 0, n_sm = 0, smem_optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        kie::dynamic_smem_limit(&smem_optin) != cudaSuccess)
      return KIE_ERR_CUDA;
    const int grid = std::min(std::min(n_sm, kMaxCtas), (int)N);

    // The rows split as the LM-head stage splits a vocabulary; the four layer
    // stages of the one-layer plan own no rows.
    kie::Shape sh{1, K, 1, 1, 64, 256, N};
    const std::vector<int2> lm = kie::partition(sh, grid, kie::ST_LM);
    int2 ranges[kie::N_STAGES * kMaxCtas] = {};
    unsigned long long off[kMaxCtas] = {};
    int maxrows = 0;
    size_t total = 0;
    for (int c = 0; c < grid; ++c) {
      ranges[kie::ST_LM * grid + c] = lm[c];
      maxrows = std::max(maxrows, lm[c].y - lm[c].x);
      off[c] = total;
      total += (size_t)(lm[c].y - lm[c].x) * K * 2;
    }

    kie::SmemLayout L{};
    L.xs_bytes = (K * 4 + 127) / 128 * 128;
    L.rowacc_rows = kie::result_slots(maxrows, K / kie::kPieceElems, kChunkBytes);
    L.resid_rows = 0;
    const int rowacc_bytes = (L.rowacc_rows * 4 + 127) / 128 * 128;
    const int bars = 2 * kie::kRingBars * 8;
    const int fixed = bars + L.xs_bytes + rowacc_bytes + kie::kEngineMisc;
    const int ring = (smem_optin - fixed) / 512 * 512;
    if (ring < 2 * kChunkBytes) return KIE_ERR_UNSUPPORTED;
    L.ring_off = 0;
    L.bar_off = ring;
    L.xs_off = L.bar_off + bars;
    L.rowacc_off = L.xs_off + L.xs_bytes;
    L.misc_off = L.rowacc_off + rowacc_bytes;
    L.total = L.misc_off + kie::kEngineMisc;

    auto* d_status = reinterpret_cast<DevStatus*>(scratch + kOffStatus);
    auto* d_layer = reinterpret_cast<LayerW*>(scratch + kOffLayer);
    auto* d_ranges = reinterpret_cast<int2*>(scratch + kOffRanges);
    auto* d_off = reinterpret_cast<unsigned long long*>(scratch + kOffPackedOff);
    auto* d_stats = reinterpret_cast<unsigned long long*>(scratch + kOffStats);
    unsigned char* d_packed = scratch + kOffPacked;

    MonoParams p{};
    p.L = 1;
    p.d = K;
    p.H = 1;
    p.KV = 1;
    p.hd = 64;
    p.F = 256;
    p.V = N;
    p.G = 1;
    p.layers = d_layer;
    p.lm_head = static_cast<const __half*>(W);
    p.ranges = d_ranges;
    p.grid = grid;
    p.ring_bytes = ring;
    p.chunk_bytes = kChunkBytes;
    p.packed = d_packed;
    p.packed_off = d_off;
    p.sm = L;
    p.status = d_status;
    p.cta_stats = d_stats;
    p.timeout_ns = 2000000000LL;
    p.poll_ns = 128;
    p.fault_cta = -1;

    // The previous call's status, layer table and counters are still in the
    // array: clear them; ranges and offsets are rewritten in full.
    DevStatus hs{};
    if (cudaMemsetAsync(d_status, 0, sizeof(DevStatus), st) != cudaSuccess ||
        cudaMemsetAsync(d_layer, 0, sizeof(LayerW), st) != cudaSuccess ||
        cudaMemsetAsync(d_stats, 0, sizeof(unsigned long long) * kie::kStatsPerCta * grid, st) !=
            cudaSuccess ||
        cudaMemcpyAsync(d_ranges, ranges, sizeof(int2) * kie::N_STAGES * grid,
                        cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(d_off, off, sizeof(unsigned long long) * grid, cudaMemcpyHostToDevice,
                        st) != cudaSuccess ||
        kie::repack_launch(p, d_packed, st) != cudaSuccess ||
        kie::gemv_configure() != cudaSuccess ||
        kie::gemv_launch(p, 1, x, y, 1, grid, L.total, st) != cudaSuccess ||
        cudaMemcpyAsync(&hs, d_status, sizeof hs, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return KIE_ERR_CUDA;
    if (hs.code != kie::DEV_OK) return hs.code == kie::DEV_TIMEOUT ? KIE_ERR_TIMEOUT : KIE_ERR_PROTOCOL;
    return KIE_OK;
  });
}

}  // extern "C"
