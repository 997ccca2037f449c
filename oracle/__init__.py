"""Oracle package: plain CPU restatement of the method, TEST INFRASTRUCTURE
ONLY (tests/, __graft_entry__.smoke() and bench.py's CPU legs).  The product
package never imports it."""
from .kvc_oracle import *  # noqa: F401,F403
from .kvc_oracle import PagedCache  # noqa: F401
from . import exans  # noqa: F401
