// Self-test of the bounded waits: the same wait routines the kernels use,
// pointed at something that never completes, with a short limit.  The probe
// must return with TSD_DEV_TIMEOUT set and leave the context usable.
//   kind 0: the mbarrier wait of the tensor-core attention kernels, on an
//           mbarrier nobody arrives on;
//   kind 1: the team barrier of the stochastic walk, on a counter whose
//           target is one arrival more than the CTA can supply;
//   kind 2: the cluster exchange of the stochastic walk, in a cluster of two
//           CTAs of which only the first takes part.
#include "cluster_xchg.cuh"
#include "sm100_ptx.cuh"
#include "team_barrier.cuh"
#include "tsd_common.cuh"

namespace tsd {

namespace {

__global__ void wait_probe_kernel(int kind, unsigned long long limit_ns, int2 *team,
                                  int32_t *dev_status)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag, sh_ok;
    if (kind == 0) {
        if (threadIdx.x == 0) {
            ptx::mbar_init(ptx::smem_addr(&bar), 1);
            abort_flag = 0;
            ptx::fence_barrier_init();
        }
        __syncthreads();
        bool ok = true;
        if (threadIdx.x == 0)
            ok = ptx::mbar_wait(ptx::smem_addr(&bar), 0, &abort_flag, limit_ns);
        if (threadIdx.x == 0 && !ok)
            flag(dev_status, TSD_DEV_TIMEOUT);
    } else {
        if (!team_barrier(team, 2, &sh_ok, limit_ns) && threadIdx.x == 0)
            flag(dev_status, TSD_DEV_TIMEOUT);
    }
}

// A cluster of two CTAs: CTA 0 enters an exchange that CTA 1 never joins,
// so its wait (two arrivals expected, its own only) runs out; both CTAs then
// meet at the cluster barrier before they exit.
__global__ void wait_probe_cluster_kernel(unsigned long long limit_ns, int32_t *dev_status)
{
    __shared__ XchgShared xs;
    xchg_init(&xs, 2);
    cluster_sync_all();
    if (cluster_ctarank() == 0) {
        if (!cluster_exchange(&xs, 2, 0, make_double2(1.0, 2.0), limit_ns) && threadIdx.x == 0)
            flag(dev_status, TSD_DEV_TIMEOUT);
    }
    cluster_sync_all();
}

}  // namespace

int launch_wait_probe(int kind, unsigned long long limit_ns, void *scratch,
                      int32_t *dev_status, cudaStream_t stream)
{
    if (kind == 2) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(32);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, wait_probe_cluster_kernel, limit_ns, dev_status) !=
            cudaSuccess) {
            (void)cudaGetLastError();
            return TSD_ERR_CUDA;
        }
        return TSD_OK;
    }
    int2 *team = static_cast<int2 *>(scratch);
    if (cudaMemsetAsync(team, 0, sizeof(int2), stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return TSD_ERR_CUDA;
    }
    wait_probe_kernel<<<1, 32, 0, stream>>>(kind, limit_ns, team, dev_status);
    TSD_LAUNCH_CHECK();
    return TSD_OK;
}

}  // namespace tsd
