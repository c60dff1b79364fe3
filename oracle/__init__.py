"""fp64 CPU oracle (test infrastructure only; see ttt_oracle.py)."""
from .ttt_oracle import (  # noqa: F401
    assoc_chunked_stream,
    assoc_recurrence_stream,
    assoc_scan,
    assoc_two_pass_stream,
    dual_form,
    dual_form_stream,
    inplace_chunks,
)
