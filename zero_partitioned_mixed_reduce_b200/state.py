"""Device memory for a plan's sharded state, allocated with PyTorch.

Marshalling only: torch allocates the buffers and copies packed inputs into
them; every step of the hot path runs in libzero_b200.so.
"""
import torch

from . import _capi as Z

HALF = {Z.ZERO_BF16: torch.bfloat16, Z.ZERO_FP16: torch.float16}


class Plan:
    """Owns a zero_plan handle and caches its layout."""

    def __init__(self, numels, layer_ids=None, R=1, dtype=Z.ZERO_BF16, tensor_align=8,
                 bucket_elems=0):
        self.handle = Z.zero_plan(numels, layer_ids, R, dtype, tensor_align, bucket_elems)
        info = Z.zero_plan_get_info(self.handle)
        self.__dict__.update(info)
        self.numels = [int(n) for n in numels]
        tensors = [Z.zero_plan_tensor(self.handle, k) for k in range(info["n_tensors"])]
        self.offsets = [t[0] for t in tensors]
        self.tensor_bucket = [t[2] for t in tensors]
        self.buckets = [Z.zero_plan_bucket(self.handle, b) for b in range(info["n_buckets"])]
        self.layers = [Z.zero_plan_layer(self.handle, l) for l in range(info["n_layers"])]

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and Z is not None and getattr(Z, "zero_plan_destroy", None) is not None:
            Z.zero_plan_destroy(h)  # (at interpreter exit the module may already be gone)
        self.handle = None

    def pack(self, flat_unpadded, out=None, fill=0):
        """Place an unpadded concatenation of the tensors into the padded flat
        layout (length T); padding gets `fill`."""
        if out is None:
            out = torch.full((self.T,), fill, dtype=flat_unpadded.dtype,
                             device=flat_unpadded.device)
        pos = 0
        for off, n in zip(self.offsets, self.numels):
            out[off:off + n].copy_(flat_unpadded[pos:pos + n])
            pos += n
        return out

    def unpack(self, flat_padded):
        return torch.cat([flat_padded[o:o + n] for o, n in zip(self.offsets, self.numels)])


class ShardedState:
    """R shards of master/m/v (fp32) and param (half), one or two sets, plus
    optional fp32 accumulators, each shard its own allocation."""

    def __init__(self, plan: Plan, sets=1, with_acc=False, device="cuda"):
        R, S = plan.R, plan.S
        self.plan, self.sets, self.device = plan, sets, device
        half = HALF[plan.dtype]
        self.master = [[torch.zeros(S, dtype=torch.float32, device=device) for _ in range(R)]
                       for _ in range(sets)]
        self.m = [[torch.zeros(S, dtype=torch.float32, device=device) for _ in range(R)]
                  for _ in range(sets)]
        self.v = [[torch.zeros(S, dtype=torch.float32, device=device) for _ in range(R)]
                  for _ in range(sets)]
        self.param = [[torch.zeros(S, dtype=half, device=device) for _ in range(R)]
                      for _ in range(sets)]
        self.acc = ([torch.zeros(S, dtype=torch.float32, device=device) for _ in range(R)]
                    if with_acc else None)
        self.handle = Z.StateHandle(
            [dict(master=self.master[k], m=self.m[k], v=self.v[k], param=self.param[k])
             for k in range(sets)], self.acc)

    def load(self, master_padded, param_padded, k=0):
        """Copy padded flat master (fp32) and param (half) of length T into set k."""
        S = self.plan.S
        for r in range(self.plan.R):
            self.master[k][r].copy_(master_padded[r * S:(r + 1) * S])
            self.param[k][r].copy_(param_padded[r * S:(r + 1) * S])
            self.m[k][r].zero_()
            self.v[k][r].zero_()

    def flat(self, field, k=0):
        """Concatenate the R shards of one field of set k (length T)."""
        return torch.cat(getattr(self, field)[k])
