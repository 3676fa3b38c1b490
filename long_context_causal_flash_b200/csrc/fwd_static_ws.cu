// gqa_attn_fwd_static_ws: the forward for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc: a plug-in running inside a host
// framework that owns all device memory and hands it no allocator, a service held to a
// fixed memory budget that forbids allocations after start-up, or a latency-critical
// path that must avoid the implicit device synchronisation an allocation can cause.
// They still own their inputs and outputs, but have nowhere to put the scratch
// workspace (status word and block-skip tables) that gqa_attn_fwd needs.  This entry
// point supplies that scratch from a fixed-size array in the library's own device
// memory, which every GPU that loads the library holds until the process exits.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kStaticWsBytes = GQA_ATTN_STATIC_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

// The scratch.  In host code this name is only a stand-in, not a device address:
// its address on the current device comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

std::mutex g_mutex;
void* g_ws_ptr[kMaxDevices] = {};

// Device address of the scratch on `dev` (which must be current); looked up once.
void* static_ws_on(int dev) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_ws_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess || ptr == nullptr) return nullptr;
    g_ws_ptr[dev] = ptr;
  }
  return g_ws_ptr[dev];
}

}  // namespace

extern "C" int gqa_attn_fwd_static_ws(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                                      int Hq, int Hkv, int64_t Lq, int64_t Lk, int d, int dtype, int mask_kind,
                                      int64_t q_pos_offset, const int32_t* segment_ids_q,
                                      const int32_t* segment_ids_kv, gqa_stream_t stream) {
  const int has_seg = segment_ids_q != nullptr && segment_ids_kv != nullptr;
  const size_t need = gqa_attn_workspace_bytes(B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, has_seg);
  if (need > kStaticWsBytes) return GQA_ERR_WORKSPACE;  // beyond the fixed scratch: no call is made
  // gqa_attn_workspace_bytes returns 0 exactly when the shape check that gqa_attn_fwd
  // runs first (check_shape in api.cu, the same function for both) fails, so passing
  // a null workspace here can only end in that shape error, never GQA_ERR_WORKSPACE.
  if (need == 0)  // a shape gqa_attn_fwd rejects: let it report which error, before any CUDA call
    return gqa_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, q_pos_offset, segment_ids_q,
                        segment_ids_kv, nullptr, 0, stream);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_LAUNCH;
  void* ws = static_ws_on(dev);
  if (!ws) return GQA_ERR_LAUNCH;
  // gqa_attn_fwd zeroes the status word itself and rewrites every table it reads.
  return gqa_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, Lq, Lk, d, dtype, mask_kind, q_pos_offset, segment_ids_q,
                      segment_ids_kv, ws, kStaticWsBytes, stream);
}
