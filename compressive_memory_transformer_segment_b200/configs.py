"""The workload shapes the layer is checked and measured on.

Shapes follow the workloads the Infini-attention pages describe: the Hugging
Face reproduction's 200M Llama and Llama-3-8B at segment 64 x rollout 16
("Hugging Face Infini-Attention 再現分析", section "重み減衰とロールアウト"),
the 300M LLaMA at 16,384 tokens ("Probing the Limits of Compressive Memory",
abstract) and contexts beyond 1M tokens ("Leave No Context Behind" explainer,
section "1M passkey retrieval の結果").  All values are synthetic.
"""

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H_q: int
    H_kv: int
    L: int
    d_k: int
    d_v: int
    seg_len: int
    dtype: str          # 'bf16' or 'f32' (q, k, v and out)
    rule: str           # 'linear' or 'delta'
    beta_range: float   # beta ~ U(-beta_range, beta_range)
    seed: int
    insert_pair: bool = False

    @property
    def T(self):
        return -(-self.L // self.seg_len)

    @property
    def tokens(self):
        return self.B * self.L

    def with_(self, **kw):
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 2, 256, 32, 32, 64, "f32", "linear", 2.0, 1000),
    "200m-linear": Workload("200m-linear", 8, 12, 12, 1024, 64, 64, 64, "bf16", "linear", 4.0, 1001),
    "200m-delta": Workload("200m-delta", 8, 12, 12, 1024, 64, 64, 64, "bf16", "delta", 4.0, 1001),
    "300m-linear": Workload("300m-linear", 4, 16, 16, 16384, 64, 64, 2048, "bf16", "linear", 4.0, 1002),
    "300m-delta": Workload("300m-delta", 4, 16, 16, 16384, 64, 64, 2048, "bf16", "delta", 4.0, 1002),
    "8b-delta": Workload("8b-delta", 2, 32, 8, 32768, 128, 128, 2048, "bf16", "delta", 4.0, 1003),
    "1m-linear": Workload("1m-linear", 1, 32, 32, 1048576, 128, 128, 2048, "bf16", "linear", 6.0, 1004,
                          insert_pair=True),
}


def algorithmic_flops(w):
    """Flops of one forward, counting only the work the method defines.

    Local attention: the causal half of Q K^T and P V, diagonal included,
    2*d*n*(n+1) per (batch, query head, segment of n rows) for d_k = d_v = d.
    Retrieval: 2*d_k*d_v + 2*d_k per token per query head.
    Update: 2*d_k*d_v + d_k per token per KV head; the delta rule adds
    2*d_k*d_v + 2*d_k more.
    """
    att = 0
    for s in range(w.T):
        n = min(w.seg_len, w.L - s * w.seg_len)
        att += (w.d_k + w.d_v) * n * (n + 1)
    att *= w.B * w.H_q
    ret = w.B * w.H_q * w.L * (2 * w.d_k * w.d_v + 2 * w.d_k)
    upd = w.B * w.H_kv * w.L * (2 * w.d_k * w.d_v + w.d_k)
    if w.rule == "delta":
        upd += w.B * w.H_kv * w.L * (2 * w.d_k * w.d_v + 2 * w.d_k)
    return att + ret + upd


def algorithmic_bytes(w):
    """q, k, v read once, out written once, M/z read once and written once."""
    e = 2 if w.dtype == "bf16" else 4
    io = (w.B * w.H_q * w.L * (w.d_k + w.d_v) + w.B * w.H_kv * w.L * (w.d_k + w.d_v)) * e
    state = 2 * 4 * w.B * w.H_kv * (w.d_k * w.d_v + w.d_k)
    return io + state
