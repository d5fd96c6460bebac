"""Device-side copies of the synthetic layer inputs (test infrastructure; the setup lives in synth.device)."""
from synth.device import bits, device_layer, fill_experts, to_dev_bf16  # noqa: F401
