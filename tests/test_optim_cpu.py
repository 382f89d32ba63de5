"""Parameter split of the hybrid optimizer (no GPU): Muon for hidden
matrices and flattened conv kernels, AdamW for embeddings, head and 1-D."""
import torch

from matrix_orthogonalizing_optimizer_step_b200.optim import split_params


class Tiny(torch.nn.Module):
    def __init__(self):
        super().__init__()
        self.wte = torch.nn.Embedding(50, 16)
        self.wpe = torch.nn.Embedding(8, 16)
        self.attn = torch.nn.Linear(16, 48)
        self.proj = torch.nn.Linear(16, 16, bias=False)
        self.ln = torch.nn.LayerNorm(16)
        self.conv = torch.nn.Conv2d(3, 16, 3)
        self.lm_head = torch.nn.Linear(16, 50, bias=False)
        self.frozen = torch.nn.Linear(4, 4)
        self.frozen.weight.requires_grad_(False)


def test_split_follows_the_rule():
    muon, adamw = split_params(Tiny().named_parameters())
    m = {n for n, _ in muon}
    a = {n for n, _ in adamw}
    assert m == {"attn.weight", "proj.weight", "conv.weight"}
    assert a == {"wte.weight", "wpe.weight", "attn.bias", "ln.weight", "ln.bias", "conv.bias",
                 "lm_head.weight", "frozen.bias"}
