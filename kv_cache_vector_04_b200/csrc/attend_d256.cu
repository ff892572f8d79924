// Launch table of the attention kernels for head dim 256 (every built format).
#include "attend_impl.cuh"

namespace tq {

cudaError_t launch_attend_d256(const Format& f, const DevTables& tb, const AttendArgs& a, bool scores,
                             cudaStream_t st)
{
#define TQ_A(DD, KB, VB, QJ) \
    if (f.kb == KB && f.vb == VB && f.qjl == QJ) return launch_attend_t<DD, KB, VB, QJ>(tb, a, scores, st);
    TQ_FORMATS_D(TQ_A, 256)
#undef TQ_A
    return cudaErrorInvalidValue;
}

}  // namespace tq
