// host.cu -- host-side helpers shared by the library's translation units
// (declared in host.h).
#include <cstdio>
#include <cstring>
#include <mutex>

#include "host.h"

namespace dsa {
namespace host {

namespace {
// ------------------------------------------------------------------ last failure text (per host thread)
thread_local char g_last_error[256] = "";

}  // namespace

void set_last_error(const char* text) { snprintf(g_last_error, sizeof g_last_error, "%s", text); }
const char* last_error_text() { return g_last_error; }

dsa_status fail(dsa_status st, const char* what, cudaError_t e) {
    if (e != cudaSuccess)
        snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
    else
        snprintf(g_last_error, sizeof g_last_error, "%s", what);
    return st;
}

namespace {

// ------------------------------------------------------------------ driver entry point (no libcuda link)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map_uncached(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
                       CUtensorMapL2promotion promo) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (i + 1 < rank) s[i] = strides_bytes[i];
    }
    return fn(map, dt, (cuuint32_t)rank, const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Encoded TMA descriptors, reused while the tensor (base pointer, shape, box)
// is the same: a small per-thread table keyed by the encoding arguments.
struct MapKey {
    const void* base;
    int dt, rank, swz;
    uint64_t dims[3], strides[2];
    uint32_t box[3];
    bool operator==(const MapKey& o) const { return memcmp(this, &o, sizeof(MapKey)) == 0; }
};

}  // namespace

bool make_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
              CUtensorMapL2promotion promo) {
    constexpr int kSlots = 8;
    thread_local MapKey keys[kSlots];
    thread_local CUtensorMap maps[kSlots];
    thread_local int used = 0, next = 0;
    MapKey k;
    memset(&k, 0, sizeof k);
    k.base = base;
    k.dt = (int)dt;
    k.rank = rank;
    k.swz = (int)swz;
    for (int i = 0; i < rank && i < 3; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
        if (i + 1 < rank) k.strides[i] = strides_bytes[i];
    }
    for (int i = 0; i < used; ++i)
        if (keys[i] == k) {
            *map = maps[i];
            return true;
        }
    if (!make_map_uncached(map, dt, rank, base, dims, strides_bytes, box, swz, promo)) return false;
    keys[next] = k;
    maps[next] = *map;
    next = (next + 1) % kSlots;
    if (used < kSlots) ++used;
    return true;
}

DevInfo dev_info() {
    static DevInfo cache[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    DevInfo di;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return di;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (cache[dev].sms > 0) return cache[dev];
    }
    cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&di.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    std::lock_guard<std::mutex> lock(mu);
    if (di.sms > 0) cache[dev] = di;
    return di;
}

// cudaFuncSetAttribute for the dynamic shared memory of `fn` on the current
// device, done once per (kernel, device, size).
cudaError_t set_smem_attr(const void* fn, int bytes) {
    struct Entry { const void* fn; int dev; int bytes; };
    static Entry done[256];
    static int n = 0;
    static std::mutex mu;
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (done[i].fn == fn && done[i].dev == dev && done[i].bytes >= bytes) return cudaSuccess;
    if (cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) return e;
    if (n < 256) done[n++] = Entry{fn, dev, bytes};
    return cudaSuccess;
}



}  // namespace host
}  // namespace dsa
