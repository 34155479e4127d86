// Self-test of the bounded waits: the same wait routines the kernels use,
// pointed at something that never completes, with a short limit.  The probe
// must return with TSD_DEV_TIMEOUT set and leave the context usable.
//   kind 0: the mbarrier wait of the tensor-core attention kernels, on an
//           mbarrier nobody arrives on;
//   kind 1: the team barrier of the stochastic walk, on a counter whose
//           target is one arrival more than the CTA can supply.
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

}  // namespace

int launch_wait_probe(int kind, unsigned long long limit_ns, void *scratch,
                      int32_t *dev_status, cudaStream_t stream)
{
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
