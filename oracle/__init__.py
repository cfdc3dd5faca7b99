"""Float64 CPU oracles of the fused IPA core, of the geometric attention
variant and its gradients, of MEET's distance-aware attention and of
backbone frames.  TEST INFRASTRUCTURE ONLY:
imported by tests/, by __graft_entry__.smoke() and by bench.py's CPU
baseline / reference arm, never by the product path.  Shares no code with
the CUDA library."""
from .ipa_dense import ipa_constants, ipa_dense, ipa_dense_blocked
from .geo_dense import geo_dense, geo_dense_blocked, softplus_stable
from .meet_dense import meet_dense, meet_logits
from .frames import frames_from_backbone
from .geo_grad import geo_grad
from .ipa_grad import ipa_grad, ipa_grad_gamma_scale
from .ipa_stats import ipa_forward_stats
from .ipa_module import ipa_module, projection_width, split_projection

__all__ = ["ipa_constants", "ipa_dense", "ipa_dense_blocked",
           "geo_dense", "geo_dense_blocked", "softplus_stable",
           "meet_dense", "meet_logits", "frames_from_backbone", "geo_grad", "ipa_grad", "ipa_grad_gamma_scale", "ipa_forward_stats",
           "ipa_module", "projection_width", "split_projection"]
