#pragma once
// Cluster geometries and the cluster launch helper.
#include "kernels_1d_cluster.cuh"
#include "launch_count.h"

namespace hyena {

using G1_128K = ClusterGeom<131072, 16, 512, 16>; // 1D, M = 262144 (16-CTA cluster)
using G2_32 = ClusterGeom<2048, 1, 64, 16>;       // 2D, 32 x 32 grid (64 x 64 padded)
using G2_64 = ClusterGeom<8192, 2, 128, 16>;      // 2D, 64 x 64
using G2_128 = ClusterGeom<32768, 4, 256, 16>;    // 2D, 128 x 128

template <typename G, typename Kern, typename... Args>
inline cudaError_t launch_cluster(Kern kern, int64_t units, cudaStream_t st, Args... args) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::SMEM);
    if (e != cudaSuccess) return e;
    if (G::C > 8) {  // 16-CTA clusters are a non-portable size
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units * G::C), 1, 1);
    cfg.blockDim = dim3(G::THREADS, 1, 1);
    cfg.dynamicSmemBytes = G::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = G::C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e != cudaSuccess) return e;
    return launched();
}

}  // namespace hyena
