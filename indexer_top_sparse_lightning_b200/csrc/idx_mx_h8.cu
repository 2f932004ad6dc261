// idx_mx_h8.cu -- indexer launchers for MXFP8 queries and keys and 8 index
// heads (D_I 64 and 128, one or two query tokens per tile).
#include "idx_launch.cuh"

namespace dsa {
namespace host {

template dsa_status launch_indexer<true, 8, 64, 1, true>(const dsa_batch*, const dsa_indexer_inputs*, int32_t*, float*, uint32_t*, uint8_t*, const IdxPlan&, cudaStream_t);
template dsa_status launch_indexer<true, 8, 64, 2, true>(const dsa_batch*, const dsa_indexer_inputs*, int32_t*, float*, uint32_t*, uint8_t*, const IdxPlan&, cudaStream_t);
template dsa_status launch_indexer<true, 8, 128, 1, true>(const dsa_batch*, const dsa_indexer_inputs*, int32_t*, float*, uint32_t*, uint8_t*, const IdxPlan&, cudaStream_t);
template dsa_status launch_indexer<true, 8, 128, 2, true>(const dsa_batch*, const dsa_indexer_inputs*, int32_t*, float*, uint32_t*, uint8_t*, const IdxPlan&, cudaStream_t);

}  // namespace host
}  // namespace dsa
