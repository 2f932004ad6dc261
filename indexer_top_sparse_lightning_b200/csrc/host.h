// host.h -- host-side helpers shared by the translation units of the library:
// failure text, TMA descriptor encoding (cached), per-device properties and
// kernel attributes, the indexer launch plan and the indexer launchers (one
// explicit instantiation per kernel variant, compiled in separate units).
// Nothing here is exported from the library.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/dsa.h"
#include "common.h"

namespace dsa {
namespace host {

// Records the failure text for dsa_last_error() (per host thread) and returns st.
dsa_status fail(dsa_status st, const char* what, cudaError_t e = cudaSuccess);
void set_last_error(const char* text);
const char* last_error_text();

// cuTensorMapEncodeTiled through the runtime's driver entry point, reusing the
// encoding while the tensor (base pointer, shape, box) is unchanged.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
              CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B);

// cudaFuncSetAttribute for the dynamic shared memory of `fn`, once per
// (kernel, device, size).
cudaError_t set_smem_attr(const void* fn, int bytes);

struct DevInfo {
    int sms = 0;
    int max_smem = 0;
};
constexpr int kMaxDevices = 64;
// Properties of the current device, queried once per device.
DevInfo dev_info();

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
// Mode-0 launches of a plan.
inline int64_t idx_launches(int64_t windows, int per_launch) { return (windows + per_launch - 1) / per_launch; }
// Bytes of the indexer's group region (sync words and publication headers).
inline size_t group_region_bytes(int sms) { return align256((size_t)sms * (size_t)group_ws_bytes(2, sms)); }

struct IdxPlan {
    int mode = 0;        // 0 grouped (query windows), 1 per-token
    int nq = 1;          // kernel NQ (tokens per window in mode 0)
    int grid = 0;        // CTAs per launch
    int seq_windows = 1; // mode 0: every sequence is one window
    int64_t windows = 0; // mode 0: windows of the batch (an upper bound unless seq_windows)
    int windows_per_launch = 0;
    int score_cap = 0;
    int smem = 0;
    size_t group_ws = 0; // bytes of group workspace per launch
};

using LaunchFn = dsa_status (*)(const dsa_batch*, const dsa_indexer_inputs*, int32_t*, float*, uint32_t*,
                                uint8_t*, const IdxPlan&, cudaStream_t);

// Launches of one indexer kernel variant (defined in idx_launch.cuh,
// instantiated in the idx_*.cu units).
template <bool FP8, int HI, int DI, int NQ, bool MX = false>
dsa_status launch_indexer(const dsa_batch* bt, const dsa_indexer_inputs* ix, int32_t* out_idx, float* out_score,
                          uint32_t* status, uint8_t* group_ws, const IdxPlan& pl, cudaStream_t stream);

}  // namespace host
}  // namespace dsa
