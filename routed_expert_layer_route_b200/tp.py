"""Channel-split tensor parallelism of one MoE layer over the ranks of a
process group.

A routed expert is a gated MLP whose channel c owns gate row c, up row c and
down column c ("Channel Selection for Mixture-of-Experts Decoding Needs No
Calibration Data", paperlayer.ai, section 2 "Background"), so the layer splits
over channels with no change to the arithmetic of a channel:

    y = sum_s w_s sum_c h_c(x) W_down[e_s][:, c]
      = sum_g ( sum_s w_s sum_{c in shard g} h_c(x) W_down[e_s][:, c] ).

Rank g of G holds channels [g*I/G, (g+1)*I/G) of every expert and a replica of
the router.  Every rank routes the token itself -- the routing is one fixed
float32 sequence on identical inputs, so every rank takes the same experts
with the same Eq. 2 weights ("Paper of the Week #3", section "The Receipt")
-- runs the layer on its channels into a float32 partial (moe_layer with the
shard's I), and one all-reduce (sum) of the partials over the group gives y.
Each rank streams 1/G of the routed experts' bytes; the collective here is
torch.distributed's (NCCL on GPUs).
"""
import torch

from . import moe

CHANNEL_ALIGN = 16  # moe_layer's shape rule: I % 16 == 0


def channel_range(I, world, rank):
    """[lo, hi) of the channels rank `rank` of `world` holds (equal shards)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d outside a world of %d" % (rank, world))
    if I % (CHANNEL_ALIGN * world):
        raise ValueError("I = %d does not split into %d shards of a multiple of %d channels"
                         % (I, world, CHANNEL_ALIGN))
    n = I // world
    return rank * n, (rank + 1) * n


def shard_weights(w_gate, w_up, w_down, rank, world):
    """This rank's channels of every expert, as contiguous copies:
    gate and up [E x I/G x d], down [E x d x I/G] (HF layout)."""
    I = w_gate.shape[1]
    lo, hi = channel_range(I, world, rank)
    return (w_gate[:, lo:hi, :].contiguous(), w_up[:, lo:hi, :].contiguous(),
            w_down[:, :, lo:hi].contiguous())


class ChannelSplitLayer:
    """One layer's shard on this rank.  With channel_major (one-token decode)
    the shard's down matrix is packed channel-major once, here."""

    def __init__(self, w_router, bias, w_gate, w_up, w_down, rank, world, group=None,
                 channel_major=False):
        self.w_router, self.bias = w_router, bias
        self.rank, self.world, self.group = rank, world, group
        self.w_gate, self.w_up, wd = shard_weights(w_gate, w_up, w_down, rank, world)
        self.channel_major = channel_major
        self.w_down = moe.moe_pack_w_down(wd) if channel_major else wd
        self.flags = moe.MOE_WDOWN_CHANNEL_MAJOR if channel_major else moe.MOE_PATH_AUTO

    @property
    def I_shard(self):
        return self.w_gate.shape[1]

    def partial(self, x, k1, k2, out, ws, topk_idx_out=None, topk_w_out=None, logits_out=None,
                stream=None):
        """This rank's float32 partial output [T x d] (no collective)."""
        moe.moe_layer(x, self.w_router, self.bias, self.w_gate, self.w_up, self.w_down, k1, k2,
                      out, ws, topk_idx_out=topk_idx_out, topk_w_out=topk_w_out,
                      logits_out=logits_out, flags=self.flags, stream=stream)

    def forward(self, x, k1, k2, y, ws, partial_buf=None, stream=None):
        """y [T x d] = the sum over the group of every rank's partial."""
        if partial_buf is None:
            partial_buf = torch.empty(y.shape, dtype=torch.float32, device=y.device)
        s = stream or torch.cuda.current_stream(y.device)
        with torch.cuda.stream(s):
            self.partial(x, k1, k2, partial_buf, ws, stream=s)
            if self.world > 1:
                torch.distributed.all_reduce(partial_buf, group=self.group)
            y.copy_(partial_buf)
        return y
