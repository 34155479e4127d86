// Tree attention on the 5th-generation tensor cores (tcgen05 / TMEM / TMA).
#include "tsd_common.cuh"

namespace tsd {

bool umma_attention_supported(const AttnArgs &) { return false; }
size_t umma_attention_workspace(const AttnArgs &, int) { return 0; }
int launch_umma_attention(const AttnArgs &, void *, size_t, int, cudaStream_t)
{
    return TSD_ERR_DTYPE;
}

}  // namespace tsd
