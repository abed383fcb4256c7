// host_cache.cu -- per-context caches of launch facts (see host_cache.h).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <vector>

#include "host_cache.h"

namespace qn {

namespace {

struct DriverCalls {
    PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const DriverCalls &driver_calls() {
    static const DriverCalls calls = [] {
        DriverCalls c;
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            c.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            c.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
        (void)cudaGetLastError();
        return c;
    }();
    return calls;
}

// Cache key: the context identity plus the device ordinal (the ordinal alone when the driver
// cannot name the context).
struct Key {
    uint64_t ctx;
    int dev;
    bool operator==(const Key &o) const { return ctx == o.ctx && dev == o.dev; }
};

cudaError_t current_key(Key *k) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    k->dev = dev;
    k->ctx = current_context_id();
    return cudaSuccess;
}

std::mutex g_lock;

struct SmEntry {
    Key key;
    int sms;
};
struct OccEntry {
    Key key;
    const void *kern;
    int threads;
    size_t smem;
    int ctas;
};
struct SmemEntry {
    Key key;
    const void *kern;
    size_t limit;
};
struct ClusterEntry {
    Key key;
    const void *kern;
    int threads, cluster;
    size_t smem;
    int n;
};
std::vector<SmEntry> g_sms;
std::vector<ClusterEntry> g_clusters;
std::vector<OccEntry> g_occ;
std::vector<SmemEntry> g_smem;

}  // namespace

uint64_t current_context_id() {
    const DriverCalls &d = driver_calls();
    if (!d.get_current || !d.get_id) return 0;
    CUcontext ctx = nullptr;
    if (d.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    unsigned long long id = 0;
    if (d.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return static_cast<uint64_t>(id) + 1;  // never 0 for a real context
}

cudaError_t device_sm_count(int *sms) {
    Key k;
    cudaError_t e = current_key(&k);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> guard(g_lock);
    for (const SmEntry &s : g_sms)
        if (s.key == k) {
            *sms = s.sms;
            return cudaSuccess;
        }
    int v = 0;
    e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, k.dev);
    if (e != cudaSuccess) return e;
    if (v <= 0) v = 1;
    if (k.ctx != 0) g_sms.push_back(SmEntry{k, v});
    *sms = v;
    return cudaSuccess;
}

cudaError_t resident_ctas(const void *kern, int threads, size_t smem, int *ctas) {
    Key k;
    cudaError_t e = current_key(&k);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> guard(g_lock);
        for (const OccEntry &o : g_occ)
            if (o.key == k && o.kern == kern && o.threads == threads && o.smem == smem) {
                *ctas = o.ctas;
                return cudaSuccess;
            }
    }
    e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return e;
    int v = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kern, threads, smem);
    if (e != cudaSuccess) return e;
    if (v <= 0) v = 1;
    std::lock_guard<std::mutex> guard(g_lock);
    if (k.ctx != 0) g_occ.push_back(OccEntry{k, kern, threads, smem, v});
    *ctas = v;
    return cudaSuccess;
}

cudaError_t resident_clusters(const void *kern, int threads, int cluster, size_t smem, int *clusters) {
    Key k;
    cudaError_t e = current_key(&k);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> guard(g_lock);
        for (const ClusterEntry &c : g_clusters)
            if (c.key == k && c.kern == kern && c.threads == threads && c.cluster == cluster && c.smem == smem) {
                *clusters = c.n;
                return cudaSuccess;
            }
    }
    e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cluster), 1, 1);
    cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    std::lock_guard<std::mutex> guard(g_lock);
    if (k.ctx != 0) g_clusters.push_back(ClusterEntry{k, kern, threads, cluster, smem, n});
    *clusters = n;
    return cudaSuccess;
}

cudaError_t ensure_smem_limit(const void *kern, size_t smem) {
    Key k;
    cudaError_t e = current_key(&k);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> guard(g_lock);
    SmemEntry *hit = nullptr;
    for (SmemEntry &s : g_smem)
        if (s.key == k && s.kern == kern) hit = &s;
    if (hit && hit->limit >= smem) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (k.ctx == 0) return cudaSuccess;  // unnamed context: set again next time
    if (hit)
        hit->limit = smem;
    else
        g_smem.push_back(SmemEntry{k, kern, smem});
    return cudaSuccess;
}

}  // namespace qn
