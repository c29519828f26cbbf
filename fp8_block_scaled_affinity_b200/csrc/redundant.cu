// Redundant experts for inference load balance (618zxw.cn news article on
// DeepSeek-V3, redundant-experts paragraph: the most heavily loaded experts
// are duplicated so that their tokens can be served by several copies).
// On one GPU the copies share the expert's weights: each copy is a group of
// the grouped GEMM with its own slice of the expert's rows and a weight
// index pointing at the expert's matrices.  Rows keep their order, so every
// output row is computed exactly as without copies; what changes is how the
// work of a hot expert is cut into groups, which is what an expert-parallel
// deployment would place on different GPUs.
//
//   moe_plan_redundant_experts (host): how many copies each expert gets;
//   moe_split_groups (device): per-copy row ranges and weight indices from
//   the permutation's expert offsets.
#include <vector>

#include "common.cuh"

namespace moe {
namespace {

// One thread per weight slot s (slots in expert order, an expert's copies
// adjacent; the shared expert is the last group).  Expert e = slot_expert[s]
// with c = off[e+1] - off[e] rows and r copies: copy j (0-based, j = s -
// first slot of e) owns rows off[e] + j*q + min(j, c mod r) onwards, where
// q = c / r; the first c mod r copies get one row more.
__global__ void split_groups_kernel(const int32_t* __restrict__ expert_offsets,
                                    const int32_t* __restrict__ replicas,
                                    const int32_t* __restrict__ slot_expert,
                                    const int32_t* __restrict__ first_slot, int n_experts,
                                    int n_slots, int32_t* __restrict__ slot_offsets,
                                    int32_t* __restrict__ slot_weight, int* dev_status) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s > n_slots) return;
    if (s == n_slots) {  // the shared expert, after every routed row
        slot_offsets[n_slots] = expert_offsets[n_experts];
        slot_offsets[n_slots + 1] = expert_offsets[n_experts + 1];
        slot_weight[n_slots] = n_experts;
        return;
    }
    int e = slot_expert[s];
    if (e < 0 || e >= n_experts) {
        set_status(dev_status, MOE_DEV_BAD_INPUT);
        e = 0;
    }
    const int r = max(1, replicas[e]);
    const int j = min(max(s - first_slot[e], 0), r - 1);
    const int c = expert_offsets[e + 1] - expert_offsets[e];
    const int q = c / r, extra = c - q * r;
    slot_offsets[s] = expert_offsets[e] + j * q + min(j, extra);
    slot_weight[s] = e;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_plan_redundant_experts(const int32_t* counts, int n_experts,
                                                  int n_extra, int32_t* replicas,
                                                  int32_t* slot_expert) {
    if (!counts || !replicas || !slot_expert) return MOE_ERR_NULL;
    if (n_experts < 1 || n_extra < 0 || n_experts + n_extra + 1 > 1040) return MOE_ERR_SHAPE;
    for (int e = 0; e < n_experts; ++e) {
        if (counts[e] < 0) return MOE_ERR_ARG;
        replicas[e] = 1;
    }
    // each extra slot to the expert whose copies carry the most rows each,
    // ceil(c / r), ties to the lower expert (compared exactly in integers)
    for (int x = 0; x < n_extra; ++x) {
        int best = 0;
        int64_t best_load = -1;
        for (int e = 0; e < n_experts; ++e) {
            const int64_t load = (int64_t(counts[e]) + replicas[e] - 1) / replicas[e];
            if (load > best_load) {
                best_load = load;
                best = e;
            }
        }
        ++replicas[best];
    }
    int s = 0;
    for (int e = 0; e < n_experts; ++e)
        for (int j = 0; j < replicas[e]; ++j) slot_expert[s++] = e;
    return MOE_OK;
}

extern "C" MOE_API int moe_split_groups(const MoeShape* shape, const int32_t* expert_offsets,
                                        const int32_t* replicas, const int32_t* slot_expert,
                                        const int32_t* first_slot, int n_extra,
                                        int32_t* slot_offsets, int32_t* slot_weight,
                                        int* dev_status, void* stream) {
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    if (!expert_offsets || !replicas || !slot_expert || !first_slot || !slot_offsets ||
        !slot_weight)
        return MOE_ERR_NULL;
    const int N = shape->n_routed;
    if (n_extra < 0 || N + n_extra + 1 > 1040) return MOE_ERR_SHAPE;
    const int n_slots = N + n_extra;
    split_groups_kernel<<<(n_slots + 1 + 255) / 256, 256, 0, as_stream(stream)>>>(
        expert_offsets, replicas, slot_expert, first_slot, N, n_slots, slot_offsets, slot_weight,
        dev_status);
    return check_launch();
}
