// idx_bf16_h64.cu -- indexer launchers for bf16 keys and 64 index heads
// (D_I 64 and 128, one or two query tokens per tile).
#include "idx_launch.cuh"

namespace dsa {
namespace host {

template dsa_status launch_indexer<false, 64, 64, 1>(const dsa_batch*, const dsa_indexer_inputs*, int32_t*, float*, uint32_t*, uint8_t*, const IdxPlan&, cudaStream_t);
template dsa_status launch_indexer<false, 64, 64, 2>(const dsa_batch*, const dsa_indexer_inputs*, int32_t*, float*, uint32_t*, uint8_t*, const IdxPlan&, cudaStream_t);
template dsa_status launch_indexer<false, 64, 128, 1>(const dsa_batch*, const dsa_indexer_inputs*, int32_t*, float*, uint32_t*, uint8_t*, const IdxPlan&, cudaStream_t);
template dsa_status launch_indexer<false, 64, 128, 2>(const dsa_batch*, const dsa_indexer_inputs*, int32_t*, float*, uint32_t*, uint8_t*, const IdxPlan&, cudaStream_t);

}  // namespace host
}  // namespace dsa
