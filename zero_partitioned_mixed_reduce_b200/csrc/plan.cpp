// Partition plan: flat layout, shards, buckets and layers (host only).
//
// Follows the inferensys "ZeRO Optimization" glossary pages: each
// data-parallel process owns one partition of the optimizer state, the
// gradients and the parameters (instruction-tuning page, ZeRO-1/2/3
// "Mechanism" bullets); small parameter groups are fused for the gradient
// reduction (legal pre-training page, "Bandwidth Optimization" bullet); a
// layer's parameters are gathered before the layer runs (same page, ZeRO-3
// "All-Gather on Demand"). The exact layout, bucket and layer rules are
// stated in include/zero_b200.h at zero_plan.
#include <limits>
#include <new>

#include "internal.h"

namespace {

int64_t next_multiple(int64_t x, int64_t m) {
    int64_t r = x % m;
    return r == 0 ? x : x + (m - r);
}

}  // namespace

extern "C" zero_status zero_plan(const int64_t* numels, const int32_t* layer_ids, int64_t n,
                                 const zero_plan_config* cfg, zero_plan_t** out) {
    return zb_guarded("zero_plan", [&]() -> zero_status {
        if (!out) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan: out is NULL");
        *out = nullptr;
        if (!numels || !cfg) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan: NULL numels or cfg");
        if (n < 1) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan: need at least one tensor");
        if (cfg->R < 1 || cfg->R > ZERO_MAX_RANKS)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan: R must be in [1, 64]");
        if (cfg->dtype != ZERO_BF16 && cfg->dtype != ZERO_FP16)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan: dtype must be ZERO_BF16 or ZERO_FP16");
        if (cfg->tensor_align < 1 || cfg->tensor_align > 4096)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan: tensor_align must be in [1, 4096]");
        if (cfg->reserved != 0) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan: reserved must be 0");

        zero_plan_t* p = new (std::nothrow) zero_plan_t();
        if (!p) return zb_fail(ZERO_ERR_OOM, "zero_plan: out of host memory");
        try {
            p->R = cfg->R;
            p->dtype = cfg->dtype;
            p->align = cfg->tensor_align;
            p->bucket_elems = cfg->bucket_elems;
            p->numel.assign(numels, numels + n);
            p->offset.resize(n);
            p->tensor_bucket.resize(n);
            p->tensor_layer.resize(n);

            // flat layout
            int64_t end = 0, total = 0;
            for (int64_t k = 0; k < n; ++k) {
                if (numels[k] < 1) {
                    delete p;
                    return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan: tensor " + std::to_string(k) +
                                                             " has numel < 1");
                }
                int64_t at = next_multiple(end, p->align);
                if (at > std::numeric_limits<int64_t>::max() - numels[k]) {
                    delete p;
                    return zb_fail(ZERO_ERR_RANGE, "zero_plan: flat length overflows");
                }
                p->offset[k] = at;
                end = at + numels[k];
                total += numels[k];
            }
            p->P = total;
            p->L = end;
            const int64_t per_rank = end / p->R + (end % p->R != 0 ? 1 : 0);
            p->S = next_multiple(per_rank, 8);
            p->T = p->S * p->R;
            // vector indices (8 elements) of the whole flat buffer are 32-bit on the device
            if (p->T / 8 >= (int64_t(1) << 31)) {
                delete p;
                return zb_fail(ZERO_ERR_RANGE, "zero_plan: padded length too large (T/8 >= 2^31)");
            }

            // buckets, formed from the last tensor backwards
            int64_t k = n - 1;
            while (k >= 0) {
                const int64_t last = k;
                int64_t count = numels[k];
                int64_t first = k;
                for (;;) {
                    if (first == 0) break;
                    if (p->bucket_elems > 0 && count + numels[first - 1] > p->bucket_elems) break;
                    --first;
                    count += numels[first];
                }
                const int64_t b = static_cast<int64_t>(p->bucket_lo.size());
                p->bucket_lo.push_back(p->offset[first]);
                p->bucket_hi.push_back(last == n - 1 ? p->T : p->offset[last + 1]);
                for (int64_t j = first; j <= last; ++j) p->tensor_bucket[j] = b;
                k = first - 1;
            }

            // layers
            if (layer_ids == nullptr) {
                for (int64_t j = 0; j < n; ++j) {
                    p->tensor_layer[j] = j;
                    p->layer_lo.push_back(p->offset[j]);
                    p->layer_hi.push_back(j + 1 < n ? p->offset[j + 1] : p->L);
                }
            } else {
                if (layer_ids[0] != 0) {
                    delete p;
                    return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan: layer_ids must start at 0");
                }
                for (int64_t j = 0; j < n; ++j) {
                    if (j > 0) {
                        const int64_t step = int64_t(layer_ids[j]) - int64_t(layer_ids[j - 1]);
                        if (step != 0 && step != 1) {
                            delete p;
                            return zb_fail(ZERO_ERR_INVALID_ARG,
                                           "zero_plan: layer_ids must step by 0 or +1 (tensor " +
                                               std::to_string(j) + ")");
                        }
                        if (step == 1) p->layer_hi.push_back(p->offset[j]);
                    }
                    if (j == 0 || layer_ids[j] != layer_ids[j - 1]) p->layer_lo.push_back(p->offset[j]);
                    p->tensor_layer[j] = layer_ids[j];
                }
                p->layer_hi.push_back(p->L);
            }
        } catch (const std::bad_alloc&) {
            delete p;
            return zb_fail(ZERO_ERR_OOM, "zero_plan: out of host memory");
        }
        *out = p;
        return ZERO_OK;
    });
}

extern "C" void zero_plan_destroy(zero_plan_t* plan) { delete plan; }

extern "C" zero_status zero_plan_get_info(const zero_plan_t* plan, zero_plan_info* info) {
    return zb_guarded("zero_plan_get_info", [&]() -> zero_status {
        if (!plan || !info) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan_get_info: NULL argument");
        info->P = plan->P;
        info->L = plan->L;
        info->S = plan->S;
        info->T = plan->T;
        info->n_tensors = static_cast<int64_t>(plan->numel.size());
        info->n_buckets = static_cast<int64_t>(plan->bucket_lo.size());
        info->n_layers = static_cast<int64_t>(plan->layer_lo.size());
        info->R = plan->R;
        info->dtype = plan->dtype;
        info->tensor_align = plan->align;
        info->reserved = 0;
        return ZERO_OK;
    });
}

extern "C" zero_status zero_plan_tensor(const zero_plan_t* plan, int64_t k, int64_t* offset,
                                        int64_t* numel, int64_t* bucket, int64_t* layer) {
    return zb_guarded("zero_plan_tensor", [&]() -> zero_status {
        if (!plan) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan_tensor: NULL plan");
        if (k < 0 || k >= static_cast<int64_t>(plan->numel.size()))
            return zb_fail(ZERO_ERR_RANGE, "zero_plan_tensor: tensor index out of range");
        if (offset) *offset = plan->offset[k];
        if (numel) *numel = plan->numel[k];
        if (bucket) *bucket = plan->tensor_bucket[k];
        if (layer) *layer = plan->tensor_layer[k];
        return ZERO_OK;
    });
}

extern "C" zero_status zero_plan_bucket(const zero_plan_t* plan, int64_t b, int64_t* lo, int64_t* hi) {
    return zb_guarded("zero_plan_bucket", [&]() -> zero_status {
        if (!plan || !lo || !hi) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan_bucket: NULL argument");
        if (b < 0 || b >= static_cast<int64_t>(plan->bucket_lo.size()))
            return zb_fail(ZERO_ERR_RANGE, "zero_plan_bucket: bucket index out of range");
        *lo = plan->bucket_lo[b];
        *hi = plan->bucket_hi[b];
        return ZERO_OK;
    });
}

extern "C" zero_status zero_plan_layer(const zero_plan_t* plan, int64_t l, int64_t* lo, int64_t* hi) {
    return zb_guarded("zero_plan_layer", [&]() -> zero_status {
        if (!plan || !lo || !hi) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan_layer: NULL argument");
        if (l < 0 || l >= static_cast<int64_t>(plan->layer_lo.size()))
            return zb_fail(ZERO_ERR_RANGE, "zero_plan_layer: layer index out of range");
        *lo = plan->layer_lo[l];
        *hi = plan->layer_hi[l];
        return ZERO_OK;
    });
}

extern "C" zero_status zero_plan_memory(const zero_plan_t* plan, int32_t stage, int64_t* bytes) {
    return zb_guarded("zero_plan_memory", [&]() -> zero_status {
        if (!plan || !bytes) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan_memory: NULL argument");
        // per element: half param 2 B, half grad 2 B, fp32 master + m + v 12 B
        const int64_t T = plan->T, S = plan->S;
        switch (stage) {
            case 0: *bytes = 16 * T; break;           // everything replicated
            case 1: *bytes = 4 * T + 12 * S; break;   // optimizer state sharded
            case 2: *bytes = 2 * T + 14 * S; break;   // + gradients sharded
            case 3: *bytes = 16 * S; break;           // + parameters sharded
            default: return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan_memory: stage must be 0..3");
        }
        return ZERO_OK;
    });
}

extern "C" zero_status zero_plan_step_tiles(const zero_plan_t* plan, int64_t* tile_elems, int64_t* tiles_per_shard,
                                            int64_t* tiles_total) {
    return zb_guarded("zero_plan_step_tiles", [&]() -> zero_status {
        if (!plan) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_plan_step_tiles: plan is NULL");
        const int64_t tps = zb::staged_tiles_per_shard(plan->S);
        if (tile_elems) *tile_elems = zb::kStagedTile;
        if (tiles_per_shard) *tiles_per_shard = tps;
        if (tiles_total) *tiles_total = tps * plan->R;
        return ZERO_OK;
    });
}
