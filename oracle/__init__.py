"""Plain, slow CPU oracle for the Windowed-MTP draft/verify attention path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (no kernels, headers, helpers or constants) and
imports nothing from it.

Sources (web pages about one paper; cited by title and section):

* "Windowed-MTP: Removing the Full-Context Draft-KV Tax at Million-Token
  Context" -- arxivlens paper view, *Abstract*, and its *Analysis* sections
  (*Results*, *Methodology*, *Technical contributions*).
* "Your Million-Token Pipeline Is Bleeding Speed You Don't Know You're Losing"
  -- readpriors.com, *What happened* (including the Figure 3 caption).
* "Does speculative decode still pay at 128K context?" -- howtospark.com case
  study, *Background*, *Method*, *Findings* ("The tax is real").

Everything here is float64 numpy (inputs are bf16 values widened exactly), or
plain Python lists for the ring buffer.  Each function names the passage it
follows.  Pins (what checks the oracle against something other than itself)
live in ``tests/test_oracle_*.py``; the list of readings taken where the pages
are silent is in the repository's design notes.

Parity status: every public function here is pinned; none is "parity
unpinned".
"""

from .attention import (  # noqa: F401
    EMPTY_LSE,
    bf16_bits_to_f64,
    attend,
    attend_rows,
    attend_prefixes,
    causal_positions,
    full_positions,
    gather_paged,
    draft_attn_full,
    draft_attn_windowed,
    draft_attn_windowed_paged,
    verify_attn,
    split_partials,
    splitkv_combine,
    window_positions,
)
from .ring import RingModel  # noqa: F401
